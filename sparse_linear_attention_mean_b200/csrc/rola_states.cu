// Linear-branch key/value states of RoLA, one CTA per (block, head, batch).
//
// SparkDiffusion write-up (0539edu.com news page), section 05: a
// rotary-positioned low-rank linear branch restores the global context of the
// blocks the sparse branch dropped.  Per block j of head h:
//   psi = phi(K_j P_h)          phi = elu + 1, padded keys -> 0
//   rho = R(t, y, x) psi        3-D rotary rotation of interleaved pairs
//   S_j = rho^T V_j  (r x d),   z_j = sum of psi over the block's keys
// and the per-head totals S = sum_j S_j, z = sum_j z_j (float64 sums).
//
// The two small contractions (K P: bs x r x d, rho^T V: r x d x bs) run on
// the tensor cores with mma.sync; rho is split into bf16 hi + lo parts so that
// rho^T V keeps ~16 mantissa bits (V is exact in bf16).  The kernel is bound
// by reading K and V once.
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {

ROLA_DEV void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
ROLA_DEV void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
ROLA_DEV void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
ROLA_DEV void cp_async16(void* dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
ROLA_DEV void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

template <int D, int R, int BS>
struct StatesSmem {
  static constexpr int KS = D + 8, PS = R + 8;
  static constexpr size_t k_off = 0;
  static constexpr size_t v_off = k_off + (size_t)BS * KS * 2;
  static constexpr size_t p_off = v_off + (size_t)BS * KS * 2;
  static constexpr size_t rh_off = p_off + (size_t)D * PS * 2;
  static constexpr size_t rl_off = rh_off + (size_t)BS * PS * 2;
  static constexpr size_t z_off = rl_off + (size_t)BS * PS * 2;
  static constexpr size_t bytes = z_off + 4 * R * sizeof(float);
};

template <int D, int R, int BS>
__global__ void __launch_bounds__(128) states_kernel(const uint16_t* __restrict__ k,
                                                     const uint16_t* __restrict__ v,
                                                     const uint16_t* __restrict__ P,
                                                     float* __restrict__ S_blk,
                                                     float* __restrict__ z_blk, int N, int H,
                                                     int Hg, int W, int nb, RopeTable rope) {
  using L = StatesSmem<D, R, BS>;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* sK = reinterpret_cast<uint16_t*>(smem + L::k_off);
  uint16_t* sV = reinterpret_cast<uint16_t*>(smem + L::v_off);
  uint16_t* sP = reinterpret_cast<uint16_t*>(smem + L::p_off);
  uint16_t* sRh = reinterpret_cast<uint16_t*>(smem + L::rh_off);
  uint16_t* sRl = reinterpret_cast<uint16_t*>(smem + L::rl_off);
  float* sZ = reinterpret_cast<float*>(smem + L::z_off);

  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const int tok0 = blk * BS;

  // ---- load K, V block rows and P_h (zero-fill tokens past N)
  constexpr int CH = D / 8;  // 16-byte chunks per row
  for (int e = tid; e < BS * CH; e += 128) {
    const int row = e / CH, ch = e % CH;
    const int tok = tok0 + row;
    const bool ok = tok < N;
    const size_t off = (((size_t)b * N + (ok ? tok : N - 1)) * H + h) * D + ch * 8;
    cp_async16(sK + row * L::KS + ch * 8, k + off, ok);
    cp_async16(sV + row * L::KS + ch * 8, v + off, ok);
  }
  constexpr int PCH = R / 8;
  for (int e = tid; e < D * PCH; e += 128) {
    const int row = e / PCH, ch = e % PCH;
    cp_async16(sP + row * L::PS + ch * 8, P + ((size_t)h * D + row) * R + ch * 8, true);
  }
  cp_async_wait_all();
  __syncthreads();

  // ---- kt = K P_h : warp w owns rows [w*RW, (w+1)*RW)
  constexpr int RW = BS / 4, MT = RW / 16, NT = R / 8;
  float acc[MT][NT][4];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D; kk += 16) {
    uint32_t a[MT][4];
#pragma unroll
    for (int mi = 0; mi < MT; ++mi)
      ldsm_x4(a[mi], sK + (warp * RW + mi * 16 + (lane & 15)) * L::KS + kk + (lane >> 4) * 8);
#pragma unroll
    for (int nj = 0; nj < NT; nj += 2) {
      uint32_t bb[4];
      ldsm_x4_t(bb, sP + (kk + (lane & 15)) * L::PS + nj * 8 + (lane >> 4) * 8);
#pragma unroll
      for (int mi = 0; mi < MT; ++mi) {
        mma_bf16_16816(acc[mi][nj], a[mi], bb[0], bb[1]);
        mma_bf16_16816(acc[mi][nj + 1], a[mi], bb[2], bb[3]);
      }
    }
  }

  // ---- psi, rho (hi/lo bf16 into shared), z partial sums
  float zp[NT][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) zp[j][0] = zp[j][1] = 0.f;
#pragma unroll
  for (int mi = 0; mi < MT; ++mi)
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = warp * RW + mi * 16 + g + half * 8;
      const int tok = tok0 + row;
      const bool ok = tok < N;
      const int pt = tok / (Hg * W), py = (tok / W) % Hg, px = tok % W;
#pragma unroll
      for (int nj = 0; nj < NT; ++nj) {
        const int col = nj * 8 + 2 * t4;
        const int pair = col >> 1;
        float p0 = ok ? phi(acc[mi][nj][2 * half]) : 0.f;
        float p1 = ok ? phi(acc[mi][nj][2 * half + 1]) : 0.f;
        zp[nj][0] += p0;
        zp[nj][1] += p1;
        const int ax = rope.axis[pair];
        const int pos = ax == 0 ? pt : (ax == 1 ? py : px);
        float sn, cs;
        rope_sincos(pos, rope.freq[pair], &sn, &cs);
        const float r0 = p0 * cs - p1 * sn;
        const float r1 = p0 * sn + p1 * cs;
        const uint32_t hi = pack_bf16(r0, r1);
        const uint32_t lo = pack_bf16(r0 - bf16_lo(hi), r1 - bf16_hi(hi));
        *reinterpret_cast<uint32_t*>(sRh + row * L::PS + col) = hi;
        *reinterpret_cast<uint32_t*>(sRl + row * L::PS + col) = lo;
      }
    }
#pragma unroll
  for (int nj = 0; nj < NT; ++nj)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float x = zp[nj][e];
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      x += __shfl_xor_sync(0xffffffffu, x, 8);
      x += __shfl_xor_sync(0xffffffffu, x, 16);
      if (g == 0) sZ[warp * R + nj * 8 + 2 * t4 + e] = x;
    }
  __syncthreads();

  const size_t state = (((size_t)b * H + h) * nb + blk);
  if (tid < R) z_blk[state * R + tid] = sZ[tid] + sZ[R + tid] + sZ[2 * R + tid] + sZ[3 * R + tid];

  // ---- S^T pieces: C[r, d] = rho^T V, warp w owns columns [w*DW, (w+1)*DW)
  constexpr int DW = D / 4, NT2 = DW / 8, MT2 = R / 16;
  float c2[MT2][NT2][4];
#pragma unroll
  for (int i = 0; i < MT2; ++i)
#pragma unroll
    for (int j = 0; j < NT2; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) c2[i][j][e] = 0.f;
#pragma unroll
  for (int kt = 0; kt < BS; kt += 16) {
    uint32_t ah[MT2][4], al[MT2][4];
    const int arow = kt + (lane & 7) + ((lane >> 4) << 3);
    const int acol = ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int mi = 0; mi < MT2; ++mi) {
      ldsm_x4_t(ah[mi], sRh + arow * L::PS + mi * 16 + acol);
      ldsm_x4_t(al[mi], sRl + arow * L::PS + mi * 16 + acol);
    }
#pragma unroll
    for (int nj = 0; nj < NT2; nj += 2) {
      uint32_t bb[4];
      ldsm_x4_t(bb, sV + (kt + (lane & 15)) * L::KS + warp * DW + nj * 8 + (lane >> 4) * 8);
#pragma unroll
      for (int mi = 0; mi < MT2; ++mi) {
        mma_bf16_16816(c2[mi][nj], ah[mi], bb[0], bb[1]);
        mma_bf16_16816(c2[mi][nj], al[mi], bb[0], bb[1]);
        mma_bf16_16816(c2[mi][nj + 1], ah[mi], bb[2], bb[3]);
        mma_bf16_16816(c2[mi][nj + 1], al[mi], bb[2], bb[3]);
      }
    }
  }
  float* Sout = S_blk + state * R * D;
#pragma unroll
  for (int mi = 0; mi < MT2; ++mi)
#pragma unroll
    for (int nj = 0; nj < NT2; ++nj) {
      const int rr = mi * 16 + g, dd = warp * DW + nj * 8 + 2 * t4;
      *reinterpret_cast<float2*>(Sout + (size_t)rr * D + dd) = make_float2(c2[mi][nj][0], c2[mi][nj][1]);
      *reinterpret_cast<float2*>(Sout + (size_t)(rr + 8) * D + dd) =
          make_float2(c2[mi][nj][2], c2[mi][nj][3]);
    }
}

// Per-head totals over blocks, summed in float64 in block order.
__global__ void __launch_bounds__(256) states_total_kernel(const float* __restrict__ S_blk,
                                                           const float* __restrict__ z_blk,
                                                           float* __restrict__ S_glb,
                                                           float* __restrict__ z_glb, int nb,
                                                           int rd, int r) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  const size_t bh = blockIdx.y;
  if (e < rd) {
    const float* p = S_blk + bh * nb * rd + e;
    double s = 0.0;
    for (int j = 0; j < nb; ++j) s += (double)p[(size_t)j * rd];
    S_glb[bh * rd + e] = (float)s;
  } else if (e < rd + r) {
    const int c = e - rd;
    const float* p = z_blk + bh * nb * r + c;
    double s = 0.0;
    for (int j = 0; j < nb; ++j) s += (double)p[(size_t)j * r];
    z_glb[bh * r + c] = (float)s;
  }
}

template <int D, int R, int BS>
static rola_status_t launch_states(const rola_shape_t* s, const uint16_t* k, const uint16_t* v,
                                   const uint16_t* P, float* S_blk, float* z_blk,
                                   const RopeTable& rope, cudaStream_t cs) {
  using L = StatesSmem<D, R, BS>;
  auto kern = states_kernel<D, R, BS>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::bytes) !=
      cudaSuccess)
    return ROLA_ERR_CUDA;
  const int nb = rola_num_blocks(s);
  kern<<<dim3(nb, s->H, s->B), 128, L::bytes, cs>>>(k, v, P, S_blk, z_blk, s->N, s->H, s->Hg, s->W,
                                                    nb, rope);
  return ROLA_OK;
}

rola_status_t launch_states_total(const rola_shape_t* s, const float* S_blk, const float* z_blk,
                                  float* S_glb, float* z_glb, cudaStream_t cs) {
  const int nb = rola_num_blocks(s);
  const int rd = s->r * s->d;
  states_total_kernel<<<dim3((rd + s->r + 255) / 256, s->B * s->H), 256, 0, cs>>>(S_blk, z_blk, S_glb,
                                                                                  z_glb, nb, rd, s->r);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

}  // namespace rola

using namespace rola;

extern "C" rola_status_t rola_block_states(const rola_shape_t* s, const uint16_t* k,
                                           const uint16_t* v, const uint16_t* P, float* S_blk,
                                           float* z_blk, float* S_glb, float* z_glb,
                                           void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!k || !v || !P || !S_blk || !z_blk || !S_glb || !z_glb) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(k, 16) || !rola_host::aligned(v, 16) || !rola_host::aligned(P, 16) ||
      !rola_host::aligned(S_blk, 16) || !rola_host::aligned(z_blk, 4) ||
      !rola_host::aligned(S_glb, 4) || !rola_host::aligned(z_glb, 4))
    return ROLA_ERR_ALIGNMENT;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (prep_kernel_supports(s)) {
    // the persistent TMA-fed pass (no pooling)
    st = launch_prep_kernel(s, nullptr, k, v, P, nullptr, nullptr, S_blk, z_blk, nullptr, cs);
    if (st != ROLA_OK) return st;
    return launch_states_total(s, S_blk, z_blk, S_glb, z_glb, cs);
  }
  RopeTable rope{};
  rola_host::rope_frequencies(s->r, s->rope_base, rope.freq, rope.axis);
  const int key = s->d * 1000000 + s->r * 1000 + s->block;
  switch (key) {
    case 128 * 1000000 + 32 * 1000 + 128: st = launch_states<128, 32, 128>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 128 * 1000000 + 16 * 1000 + 128: st = launch_states<128, 16, 128>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 128 * 1000000 + 32 * 1000 + 64: st = launch_states<128, 32, 64>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 128 * 1000000 + 16 * 1000 + 64: st = launch_states<128, 16, 64>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 64 * 1000000 + 32 * 1000 + 128: st = launch_states<64, 32, 128>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 64 * 1000000 + 16 * 1000 + 128: st = launch_states<64, 16, 128>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 64 * 1000000 + 32 * 1000 + 64: st = launch_states<64, 32, 64>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    case 64 * 1000000 + 16 * 1000 + 64: st = launch_states<64, 16, 64>(s, k, v, P, S_blk, z_blk, rope, cs); break;
    default: return ROLA_ERR_UNSUPPORTED;
  }
  if (st != ROLA_OK) return st;
  return launch_states_total(s, S_blk, z_blk, S_glb, z_glb, cs);
}
