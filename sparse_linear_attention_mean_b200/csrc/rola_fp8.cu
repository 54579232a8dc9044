// W8A8 FP8 E4M3 projections.
//
// SparkDiffusion write-up (0539edu.com news page), section 07: the linear
// projections of attention and FFN are quantised to W8A8 FP8 E4M3 and the
// activation scaling and type conversion are fused, to cut memory traffic
// and kernel launches.  Scales: per token for activations, per output
// channel for weights, s = amax / 448; codes E4M3(x * (448 / amax)) with the
// reciprocal and the product each rounded to float32, converted with
// round-to-nearest-even and saturation (cvt.rn.satfinite).
#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {

ROLA_DEV uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

ROLA_DEV float block_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) red[0] = v;
  }
  __syncthreads();
  return red[0];
}

// One CTA per row; the row stays in registers between the amax pass and the
// cast (read once from HBM).  T = bf16 bits (uint16_t) or float.
template <typename T, int MAXV>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ x,
                                                         uint8_t* __restrict__ q,
                                                         float* __restrict__ scale, int K) {
  __shared__ float red[32];
  const size_t row = blockIdx.x;
  constexpr int EPV = 8;  // elements per vector
  const int nvec = K / EPV;
  float v[MAXV][EPV];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c < nvec) {
      if constexpr (sizeof(T) == 2) {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(x + row * K) + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[i][2 * e] = bf16_lo(w[e]);
          v[i][2 * e + 1] = bf16_hi(w[e]);
        }
      } else {
        const float4 a = __ldg(reinterpret_cast<const float4*>(x + row * K) + 2 * c);
        const float4 b = __ldg(reinterpret_cast<const float4*>(x + row * K) + 2 * c + 1);
        v[i][0] = a.x; v[i][1] = a.y; v[i][2] = a.z; v[i][3] = a.w;
        v[i][4] = b.x; v[i][5] = b.y; v[i][6] = b.z; v[i][7] = b.w;
      }
#pragma unroll
      for (int e = 0; e < EPV; ++e) amax = fmaxf(amax, fabsf(v[i][e]));
    }
  }
  amax = block_max(amax, red);
  const float inv = amax > 0.f ? __fdiv_rn(448.f, amax) : 448.f;
  if (threadIdx.x == 0) scale[row] = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int c = threadIdx.x + i * 256;
    if (c < nvec) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        lo |= e4m3x2(__fmul_rn(v[i][e], inv), __fmul_rn(v[i][e + 1], inv)) << (8 * e);
        hi |= e4m3x2(__fmul_rn(v[i][4 + e], inv), __fmul_rn(v[i][5 + e], inv)) << (8 * e);
      }
      reinterpret_cast<uint2*>(q + row * K)[c] = make_uint2(lo, hi);
    }
  }
}

template <typename T>
static rola_status_t launch_quant(int M, int K, const T* x, uint8_t* q, float* s, cudaStream_t cs) {
  const int nvec = K / 8;
  const int per = (nvec + 255) / 256;
  if (per <= 1) quant_rows_kernel<T, 1><<<M, 256, 0, cs>>>(x, q, s, K);
  else if (per <= 2) quant_rows_kernel<T, 2><<<M, 256, 0, cs>>>(x, q, s, K);
  else if (per <= 4) quant_rows_kernel<T, 4><<<M, 256, 0, cs>>>(x, q, s, K);
  else if (per <= 8) quant_rows_kernel<T, 8><<<M, 256, 0, cs>>>(x, q, s, K);
  else return ROLA_ERR_UNSUPPORTED;
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

}  // namespace rola

using namespace rola;

extern "C" rola_status_t fp8_quantize_rows_bf16(int32_t M, int32_t K, const uint16_t* x,
                                                uint8_t* x_q, float* scale, void* stream) {
  if (M < 1 || K < 16 || K % 16 != 0 || !x || !x_q || !scale) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(x, 16) || !rola_host::aligned(x_q, 8)) return ROLA_ERR_ALIGNMENT;
  return launch_quant<uint16_t>(M, K, x, x_q, scale, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" rola_status_t fp8_quantize_weight(int32_t N, int32_t K, const float* w, uint8_t* w_q,
                                             float* w_scale, void* stream) {
  if (N < 1 || K < 16 || K % 16 != 0 || !w || !w_q || !w_scale) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(w, 16) || !rola_host::aligned(w_q, 8)) return ROLA_ERR_ALIGNMENT;
  return launch_quant<float>(N, K, w, w_q, w_scale, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" size_t fp8_linear_workspace_bytes(int32_t M, int32_t K) {
  if (M < 1 || K < 1) return 0;
  return rola_internal::round_up((size_t)M * K, 256) + rola_internal::round_up((size_t)M * 4, 256);
}

extern "C" rola_status_t fp8_linear_w8a8(int32_t M, int32_t N, int32_t K, const uint16_t* x,
                                         const uint8_t* w_q, const float* w_scale, uint16_t* y,
                                         void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  if (M < 1 || N < 1 || K < 1 || !x || !w_q || !w_scale || !y) return ROLA_ERR_INVALID_ARG;
  const size_t need = fp8_linear_workspace_bytes(M, K);
  if (!ws || ws_bytes < need || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  uint8_t* xq = reinterpret_cast<uint8_t*>(ws);
  float* xs = reinterpret_cast<float*>(xq + rola_internal::round_up((size_t)M * K, 256));
  rola_status_t st = fp8_quantize_rows_bf16(M, K, x, xq, xs, stream);
  if (st != ROLA_OK) return st;
  return fp8_gemm_w8a8(M, N, K, xq, xs, w_q, w_scale, y, dev_err, stream);
}

// ---------------------------------------------------------------- FFN
// Workspace of fp8_ffn_w8a8: codes and scales of x, the bf16 hidden
// activation, and its codes and scales.
struct FfnWs {
  size_t xq, xs, h, hq, hs, total;
};
static FfnWs ffn_ws(int32_t M, int32_t D, int32_t F) {
  using rola_internal::round_up;
  FfnWs w{};
  size_t off = 0;
  w.xq = off; off += round_up((size_t)M * D, 256);
  w.xs = off; off += round_up((size_t)M * 4, 256);
  w.h = off;  off += round_up((size_t)M * F * 2, 256);
  w.hq = off; off += round_up((size_t)M * F, 256);
  w.hs = off; off += round_up((size_t)M * 4, 256);
  w.total = off;
  return w;
}

extern "C" size_t fp8_ffn_workspace_bytes(int32_t M, int32_t D, int32_t F) {
  if (M < 1 || D < 1 || F < 1) return 0;
  return ffn_ws(M, D, F).total;
}

extern "C" rola_status_t fp8_ffn_w8a8(int32_t M, int32_t D, int32_t F, const uint16_t* x,
                                      const uint8_t* w1_q, const float* w1_scale,
                                      const uint8_t* w2_q, const float* w2_scale, uint16_t* y,
                                      void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  if (M < 1 || D < 1 || F < 1 || !x || !w1_q || !w1_scale || !w2_q || !w2_scale || !y)
    return ROLA_ERR_INVALID_ARG;
  if (D % 32 != 0 || F % 32 != 0) return ROLA_ERR_INVALID_ARG;
  const FfnWs L = ffn_ws(M, D, F);
  if (!ws || ws_bytes < L.total || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  char* base = reinterpret_cast<char*>(ws);
  uint8_t* xq = reinterpret_cast<uint8_t*>(base + L.xq);
  float* xs = reinterpret_cast<float*>(base + L.xs);
  uint16_t* h = reinterpret_cast<uint16_t*>(base + L.h);
  uint8_t* hq = reinterpret_cast<uint8_t*>(base + L.hq);
  float* hs = reinterpret_cast<float*>(base + L.hs);
  rola_status_t st = fp8_quantize_rows_bf16(M, D, x, xq, xs, stream);
  if (st != ROLA_OK) return st;
  st = fp8_gemm_w8a8_act(M, F, D, xq, xs, w1_q, w1_scale, ROLA_ACT_GELU_TANH, h, dev_err, stream);
  if (st != ROLA_OK) return st;
  st = fp8_quantize_rows_bf16(M, F, h, hq, hs, stream);
  if (st != ROLA_OK) return st;
  return fp8_gemm_w8a8(M, D, F, hq, hs, w2_q, w2_scale, y, dev_err, stream);
}
