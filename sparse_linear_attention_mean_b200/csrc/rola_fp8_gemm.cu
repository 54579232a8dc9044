// W8A8 FP8 E4M3 GEMM on the fifth-generation tensor cores.
//
// SparkDiffusion write-up (0539edu.com news page), section 07: the attention
// and FFN projections run as W8A8 FP8 E4M3 GEMMs with the activation scale
// folded into the product.  This kernel computes
//   y[m, n] = bf16( (sum_k dec(x_q[m, k]) * dec(w_q[n, k])) * x_scale[m] * w_scale[n] )
// for row-major x_q [M, K] and w_q [N, K] (both K-major), y [M, N] bf16.
//
// Design (one persistent CTA per SM, 192 threads):
//   warp 0      TMA producer: 128 x 128-byte A tiles and 256 x 128-byte B
//               tiles (128-byte swizzle) into a 4-stage ring (48 KB a stage);
//   warp 1      MMA issuer: tcgen05.mma kind::f8f6f4, M = 128, N = 256,
//               K = 32 per instruction, fp32 accumulators in tensor memory,
//               two 256-column accumulators so that the epilogue of one tile
//               overlaps the main loop of the next;
//   warps 2-5   epilogue: tcgen05.ld of their 32-lane quarter, scale by
//               x_scale[m] * w_scale[n], optionally apply GELU (tanh form,
//               the FFN's up projection), round to bf16, store.
// Tiles are walked n-fastest so that the CTAs resident at one time share a
// few 128-row panels of x_q in L2 while all of w_q stays L2-resident.
// Every wait is bounded; on a timeout the CTA drains its copies and MMAs,
// frees tensor memory and reports ROLA_DEVERR_TIMEOUT in *dev_err.
#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {
namespace fp8g {

constexpr int BM = 128, BN = 256, BK = 128;  // BK in elements (= bytes)
constexpr int S = 4;                         // ring stages
constexpr uint32_t A_BYTES = BM * BK, B_BYTES = BN * BK, STAGE = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr int kEpiWarps = 4;

struct Misc {
  uint64_t full[S], empty[S], acc_full[2], acc_empty[2], mma_final;
  uint32_t tmem;
  int abort;
};
constexpr size_t kMiscOff = (size_t)S * STAGE;
constexpr size_t kSmem = kMiscOff + sizeof(Misc) + 1024;  // + alignment slack

struct Params {
  int M, N, K;
  int tiles_n, tiles, kblocks;
  const float* x_scale;
  const float* w_scale;
  uint16_t* y;
  int32_t* dev_err;
  int act;  // ROLA_ACT_NONE or ROLA_ACT_GELU_TANH
};

// GELU in its tanh form, 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))), in
// float32 with the CUDA math library's tanhf.
ROLA_DEV float gelu_tanh(float u) {
  const float kC = 0.7978845608028654f;  // sqrt(2 / pi)
  return 0.5f * u * (1.f + tanhf(kC * fmaf(0.044715f * u, u * u, u)));
}

__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const Params p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte swizzle atoms
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Misc& M = *reinterpret_cast<Misc*>(smem + kMiscOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &M.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(&M.full[i], 1);
      mbar_init(&M.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&M.acc_full[i], 1);
      mbar_init(&M.acc_empty[i], kEpiWarps);
    }
    mbar_init(&M.mma_final, 1);
    M.abort = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&M.tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = M.tmem;

  if (warp == 0) {
    // ================================================================ producer
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const uint32_t st = it % S;
          if (it >= (uint32_t)S && !(ok = mbar_wait(&M.empty[st], ((it / S) - 1) & 1, abort))) break;
          uint8_t* a = smem + st * STAGE;
          mbar_expect_tx(&M.full[st], STAGE);
          tma_load_2d(a, &tmA, &M.full[st], kb * BK, m0);
          tma_load_2d(a + A_BYTES, &tmB, &M.full[st], kb * BK, n0);
        }
      }
      if (!ok) {
        // drain: the last S issued copies may still be landing
        int no_abort = 0;
        const uint32_t first = it > (uint32_t)S ? it - S : 0;
        for (uint32_t j = first; j < it; ++j) mbar_wait(&M.full[j % S], (j / S) & 1, &no_abort);
      }
    }
  } else if (warp == 1) {
    // ================================================================ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = instr_desc(kFmtE4M3, kFmtE4M3, false, false, BM, BN);
      const uint32_t sbase = smem_u32(smem);
      uint32_t it = 0, lt = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x, ++lt) {
        const uint32_t buf = lt & 1;
        if (lt >= 2 && !(ok = mbar_wait(&M.acc_empty[buf], ((lt >> 1) - 1) & 1, abort))) break;
        tc_fence_after();
        const uint32_t d = tm + buf * BN;
        for (int kb = 0; kb < p.kblocks; ++kb, ++it) {
          const uint32_t st = it % S;
          if (!(ok = mbar_wait(&M.full[st], (it / S) & 1, abort))) break;
          tc_fence_after();
          const uint32_t a = sbase + st * STAGE, b = a + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk) {
            // K-major, 128-byte swizzle: 8-row groups 1024 B apart, K step of
            // 32 bytes inside the swizzle atom
            const uint64_t ad = smem_desc(a + kk * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = smem_desc(b + kk * 32, 16, 1024, kSwizzle128B);
            mma_ss(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u, true);
          }
          mma_commit(&M.empty[st]);
        }
        if (!ok) break;
        mma_commit(&M.acc_full[buf]);
      }
      mma_commit(&M.mma_final);
      int no_abort = 0;
      mbar_wait(&M.mma_final, 0, &no_abort);
      if (no_abort) *abort = 1;
    }
  } else {
    // ================================================================ epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    uint32_t lt = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x, ++lt) {
      const uint32_t buf = lt & 1;
      const bool ok = mbar_wait(&M.acc_full[buf], (lt >> 1) & 1, abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
      const int m = m0 + quarter * 32 + lane;
      const float xs = m < p.M ? __ldg(p.x_scale + m) : 0.f;
      const uint32_t taddr = tm + ((uint32_t)(quarter * 32) << 16) + buf * BN;
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(taddr + c * 32, r);
        tmem_wait_ld();
        if (c == BN / 32 - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&M.acc_empty[buf]);
        }
        const int n = n0 + c * 32;
        if (n >= p.N) continue;
        float wsc[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 w4 = __ldg(reinterpret_cast<const float4*>(p.w_scale + n) + j);
          wsc[4 * j] = w4.x * xs;
          wsc[4 * j + 1] = w4.y * xs;
          wsc[4 * j + 2] = w4.z * xs;
          wsc[4 * j + 3] = w4.w * xs;
        }
        if (m < p.M) {
          uint4* dst = reinterpret_cast<uint4*>(p.y + (size_t)m * p.N + n);
          if (p.act == ROLA_ACT_GELU_TANH) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              r[j] = __float_as_uint(gelu_tanh(__uint_as_float(r[j]) * wsc[j]));
#pragma unroll
            for (int j = 0; j < 32; ++j) wsc[j] = 1.f;
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            uint4 o;
            o.x = pack_bf16(__uint_as_float(r[8 * j + 0]) * wsc[8 * j + 0], __uint_as_float(r[8 * j + 1]) * wsc[8 * j + 1]);
            o.y = pack_bf16(__uint_as_float(r[8 * j + 2]) * wsc[8 * j + 2], __uint_as_float(r[8 * j + 3]) * wsc[8 * j + 3]);
            o.z = pack_bf16(__uint_as_float(r[8 * j + 4]) * wsc[8 * j + 4], __uint_as_float(r[8 * j + 5]) * wsc[8 * j + 5]);
            o.w = pack_bf16(__uint_as_float(r[8 * j + 6]) * wsc[8 * j + 6], __uint_as_float(r[8 * j + 7]) * wsc[8 * j + 7]);
            dst[j] = o;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  if (threadIdx.x == 0 && p.dev_err && M.abort) atomicOr(p.dev_err, ROLA_DEVERR_TIMEOUT);
}

// 2-D TMA map over a row-major [rows, K] byte matrix, box of 128 bytes x
// box_rows rows, 128-byte swizzle, zero fill outside.
static bool make_fp8_map(CUtensorMap* m, const void* base, int rows, int K, int box_rows) {
  auto enc = rola_host::encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)K};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fp8g
}  // namespace rola

extern "C" rola_status_t fp8_gemm_w8a8_act(int32_t M, int32_t N, int32_t K, const uint8_t* x_q,
                                           const float* x_scale, const uint8_t* w_q,
                                           const float* w_scale, int32_t act, uint16_t* y,
                                           int32_t* dev_err, void* stream) {
  using namespace rola::fp8g;
  if (M < 1 || N < 32 || K < 16 || N % 32 != 0 || K % 16 != 0) return ROLA_ERR_INVALID_ARG;
  if (act != ROLA_ACT_NONE && act != ROLA_ACT_GELU_TANH) return ROLA_ERR_INVALID_ARG;
  if (!x_q || !x_scale || !w_q || !w_scale || !y) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(x_q, 16) || !rola_host::aligned(w_q, 16) || !rola_host::aligned(y, 16) ||
      !rola_host::aligned(w_scale, 16) || !rola_host::aligned(x_scale, 4))
    return ROLA_ERR_ALIGNMENT;
  CUtensorMap ma, mb;
  if (!make_fp8_map(&ma, x_q, M, K, BM) || !make_fp8_map(&mb, w_q, N, K, BN)) return ROLA_ERR_CUDA;
  Params prm{};
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.tiles_n = (N + BN - 1) / BN;
  const long long tiles = (long long)((M + BM - 1) / BM) * prm.tiles_n;
  if (tiles > 0x7fffffffLL) return ROLA_ERR_UNSUPPORTED;
  prm.tiles = (int)tiles;
  prm.kblocks = (K + BK - 1) / BK;
  prm.x_scale = x_scale;
  prm.w_scale = w_scale;
  prm.y = y;
  prm.dev_err = dev_err;
  prm.act = act;
  if (cudaFuncSetAttribute(fp8_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem) !=
      cudaSuccess)
    return ROLA_ERR_CUDA;
  const int nsm = rola_host::sm_count();
  const int grid = prm.tiles < nsm ? prm.tiles : nsm;
  fp8_gemm_kernel<<<grid, kThreads, kSmem, reinterpret_cast<cudaStream_t>(stream)>>>(ma, mb, prm);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

extern "C" rola_status_t fp8_gemm_w8a8(int32_t M, int32_t N, int32_t K, const uint8_t* x_q,
                                       const float* x_scale, const uint8_t* w_q,
                                       const float* w_scale, uint16_t* y, int32_t* dev_err,
                                       void* stream) {
  return fp8_gemm_w8a8_act(M, N, K, x_q, x_scale, w_q, w_scale, ROLA_ACT_NONE, y, dev_err, stream);
}
