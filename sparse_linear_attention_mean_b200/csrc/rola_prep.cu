// One pass over q, k and v for d = 128 and 128-token blocks: the float64
// block means of q and k that the selector scores, and the linear-branch
// states of every block, read from HBM once.
//
// SparkDiffusion write-up (0539edu.com news page), section 05: the sparse
// branch keeps the important query-key blocks (selected here from block
// means), and a rotary low-rank linear branch restores the dropped context
// (per-block states S_j = rho^T V, z_j = sum psi, rho = R(t, y, x) phi(K P_h)).
//
// Persistent CTAs (256 threads, two per SM) walk (batch, head, block) items.
// Thread 0 TMA-loads an item's k and v tiles (128-byte swizzle) and every
// thread loads its share of its q tile straight into registers while the
// previous item is still being computed: k and q once the previous item's
// pooling has consumed them, v once its state product has.  Per item:
//   * K P_h with mma.sync (first: it needs only the k tile, so the q loads
//     have this long to land);
//   * block sums of q and k over the valid tokens in float64 (exact for bf16;
//     rows past N are zero), divided by the count;
//   * psi = phi(K P_h), rho = rotation by a per-CTA cos/sin table of the 3-D
//     rotary angles, written as bf16 hi + lo;
//   * S_j^T = V^T rho with mma.sync (hi and lo parts), z_j = sum of psi.
// The kernel is bound by HBM: 96 KB read and ~16.5 KB written per item.
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {
namespace prep {

constexpr int kThreads = 256;
constexpr int D = 128, BS = 128;
constexpr uint32_t TILE = BS * D * 2;  // 32 KB
constexpr int kTabCap = 1024;

template <int R>
struct Layout {
  static constexpr uint32_t stage_bytes = 2 * TILE;  // k, v
  static constexpr int PS = R + 8;                   // padded row of P_h and rho (bf16)
  static constexpr uint32_t RHO_BYTES = BS * PS * 2;  // one of hi / lo
  // the pooling partials [8 warps][q, k][128] float64 share this buffer with
  // rho (written once the partials are consumed)
  static constexpr uint32_t PART_BYTES = 8 * 2 * D * 8;
  static constexpr uint32_t rho_off = stage_bytes;
  static constexpr uint32_t pt_off = rho_off + (2 * RHO_BYTES > PART_BYTES ? 2 * RHO_BYTES : PART_BYTES);
  static constexpr uint32_t misc_off = pt_off + D * PS * 2;
};

struct Misc {
  uint64_t full_k, full_v;
  int abort;
  int cur_h;
  float zpart[8][32];
  float2 tab[kTabCap];
};

struct Params {
  int B, H, N, nb, Hg, W, items;
  int do_pool;
  const uint16_t* q;  // [B, N, H, d] bf16 (pooling only)
  double* qbar;  // [B, H, nb, d] float64, or null
  double* kbar;
  const uint16_t* P;
  float* S_blk;
  float* z_blk;
  int32_t* dev_err;
  RopeTable rope;
  int tab_base[16], tab_stride[16], tab_first[17];
  int tab_entries;  // cos/sin table entries (the table always fits: see prep_kernel_supports)
};

ROLA_DEV void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
ROLA_DEV void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
ROLA_DEV void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Byte offset of element (row, col) of a [128 x 128] bf16 tile stored as two
// 64-column atoms with the TMA 128-byte swizzle.
ROLA_DEV uint32_t sw_off(int row, int col) {
  return (uint32_t)((col >> 6) * (BS * 128) + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) +
                    (col & 7) * 2);
}

// bf16 -> float64 times 2^-896, exactly: the bf16 sign, exponent and
// mantissa bits go to their places in the high word of a float64, whose
// exponent bias is 1023 instead of 127 (denormals map to denormals).  This
// keeps the conversion on the integer pipe; the block sums are multiplied by
// 2^896 at the end, which is exact.
ROLA_DEV double bf16lo_f64s(uint32_t w) {
  return __hiloint2double((int)(((w << 16) & 0x80000000u) | ((w << 13) & 0x0fffe000u)), 0);
}
ROLA_DEV double bf16hi_f64s(uint32_t w) {
  return __hiloint2double((int)((w & 0x80000000u) | ((w >> 3) & 0x0fffe000u)), 0);
}
constexpr double kTwo896 = 0x1p896;

template <int R>
__global__ void __launch_bounds__(kThreads, 2)
    rola_prep_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const Params p) {
  using Ly = Layout<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& M = *reinterpret_cast<Misc*>(smem + Ly::misc_off);
  uint16_t* sP = reinterpret_cast<uint16_t*>(smem + Ly::pt_off);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  // each CTA takes a contiguous run of items (consecutive blocks of one head,
  // so that P_h rarely changes)
  const int per_cta = (p.items + (int)gridDim.x - 1) / (int)gridDim.x;
  const int first_item = (int)blockIdx.x * per_cta;
  const int my_items = max(0, min(per_cta, p.items - first_item));

  if (tid == 0) {
    mbar_init(&M.full_k, 1);
    mbar_init(&M.full_v, 1);
    M.abort = 0;
    M.cur_h = -1;
    fence_barrier_init();
  }
  for (int e = tid; e < p.tab_entries; e += kThreads) {
    int pr = 0;
    while (pr + 1 < R / 2 && e >= p.tab_first[pr + 1]) ++pr;
    const int pos = e - p.tab_first[pr];
    float sn, cs;
    rope_sincos(pos, p.rope.freq[pr], &sn, &cs);
    M.tab[p.tab_base[pr] + pos * p.tab_stride[pr]] = make_float2(cs, sn);
  }
  __syncthreads();
  volatile int* abort = &M.abort;

  auto decode = [&](int it, int& b, int& h, int& blk) {
    const int id = first_item + it;
    blk = id % p.nb;
    h = (id / p.nb) % p.H;
    b = id / (p.nb * p.H);
  };
  // The k and v tiles of an item go to their buffers as soon as the previous
  // item is done with them: k after its pooling, v after its state product,
  // so that each copy overlaps the rest of the previous item.
  auto issue_k = [&](int it) {
    int b, h, blk;
    decode(it, b, h, blk);
    mbar_expect_tx(&M.full_k, TILE);
    for (int ka = 0; ka < 2; ++ka) tma_load_4d(smem + ka * (BS * 128), &tmK, &M.full_k, ka * 64, h, blk * BS, b);
  };
  auto issue_v = [&](int it) {
    int b, h, blk;
    decode(it, b, h, blk);
    mbar_expect_tx(&M.full_v, TILE);
    for (int ka = 0; ka < 2; ++ka)
      tma_load_4d(smem + TILE + ka * (BS * 128), &tmV, &M.full_v, ka * 64, h, blk * BS, b);
  };
  // pooling: thread = (row group rg of rows rg + 16 i, 8-channel chunk c8)
  const int rg = tid >> 4, c8 = tid & 15;
  double* part = reinterpret_cast<double*>(smem + Ly::rho_off);  // [8][2][D]
  // this thread's share of an item's q tile, straight into registers (it
  // is loaded for the next item as soon as this item's pooling is done)
  uint4 qv[8];
  auto load_q = [&](int it) {
    int b, h, blk;
    decode(it, b, h, blk);
    const int tok0 = blk * BS, valid = min(BS, p.N - tok0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int row = rg + 16 * i;
      qv[i] = row < valid ? __ldg(reinterpret_cast<const uint4*>(
                                p.q + (((size_t)b * p.N + tok0 + row) * p.H + h) * D + c8 * 8))
                          : make_uint4(0, 0, 0, 0);
    }
  };
  if (tid == 0 && my_items > 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    issue_k(0);
    issue_v(0);
  }
  if (p.do_pool && my_items > 0) load_q(0);
  int k_issued = my_items > 0 ? 1 : 0, v_issued = k_issued;  // copies issued (thread 0's count)

  bool ok = true;
  int it = 0;
  for (; ok && it < my_items; ++it) {
    int b, h, blk;
    decode(it, b, h, blk);
    const size_t bh = (size_t)b * p.H + h;
    const int tok0 = blk * BS;
    const int valid = min(BS, p.N - tok0);
    uint8_t* sk = smem;
    uint8_t* sv = sk + TILE;
    // P_h (rows d, padded) when the head changes
    if (h != M.cur_h) {
      for (int e = tid; e < D * (R / 8); e += kThreads) {
        const int row = e / (R / 8), ch = e % (R / 8);
        *reinterpret_cast<uint4*>(sP + row * Ly::PS + ch * 8) =
            *reinterpret_cast<const uint4*>(p.P + ((size_t)h * D + row) * R + ch * 8);
      }
      __syncthreads();
      if (tid == 0) M.cur_h = h;
    }
    if (!(ok = __syncthreads_and(mbar_wait(&M.full_k, it & 1, abort)))) break;

    // ---- kt = K P_h : warp w owns token rows [16w, 16w + 16)
    constexpr int NT = R / 8;
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
    {
      const uint32_t kbase = smem_u32(sk), pbase = smem_u32(sP);
      const int arow = warp * 16 + (lane & 15);
#pragma unroll
      for (int kk = 0; kk < D; kk += 16) {
        uint32_t a[4];
        ldsm_x4(a, kbase + sw_off(arow, kk + (lane >> 4) * 8));
#pragma unroll
        for (int nj = 0; nj < NT; nj += 2) {
          uint32_t bb[4];
          ldsm_x4_t(bb, pbase + ((kk + (lane & 15)) * Ly::PS + nj * 8 + (lane >> 4) * 8) * 2);
          mma16816(acc[nj], a, bb[0], bb[1]);
          mma16816(acc[nj + 1], a, bb[2], bb[3]);
        }
      }
    }
    // ---- block sums of q and k (float64, scaled by 2^-896: the bf16 sums are
    // exact); rows past N are zero in both (q not loaded, k zero-filled by
    // the copy)
    if (p.do_pool) {
      double aq[8], ak[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) aq[e] = ak[e] = 0.0;
      const uint32_t koff = (uint32_t)((c8 >> 3) * (BS * 128) + rg * 128 + (((c8 & 7) ^ (rg & 7)) << 4));
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 kw = *reinterpret_cast<const uint4*>(sk + koff + i * 16 * 128);
        const uint32_t qa[4] = {qv[i].x, qv[i].y, qv[i].z, qv[i].w};
        const uint32_t ka[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          aq[2 * e] += bf16lo_f64s(qa[e]);
          aq[2 * e + 1] += bf16hi_f64s(qa[e]);
          ak[2 * e] += bf16lo_f64s(ka[e]);
          ak[2 * e + 1] += bf16hi_f64s(ka[e]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        aq[e] += __shfl_xor_sync(0xffffffffu, aq[e], 16);
        ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], 16);
      }
      if (lane < 16) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          part[(warp * 2 + 0) * D + c8 * 8 + e] = aq[e];
          part[(warp * 2 + 1) * D + c8 * 8 + e] = ak[e];
        }
      }
    }

    __syncthreads();  // pooling partials complete; k and this thread's q are consumed
    if (it + 1 < my_items) {
      if (tid == 0) {
        issue_k(it + 1);
        ++k_issued;
      }
      if (p.do_pool) load_q(it + 1);
    }
    if (p.do_pool) {
      const int tile = tid >> 7, c = tid & 127;
      double acc2 = 0.0;
#pragma unroll
      for (int w = 0; w < 8; ++w) acc2 += part[(w * 2 + tile) * D + c];
      double* dst = tile == 0 ? p.qbar : p.kbar;
      dst[(bh * p.nb + blk) * D + c] = (acc2 * kTwo896) / (double)valid;
    }
    __syncthreads();  // partials consumed: rho goes over them

    // ---- psi, rho (hi / lo bf16), partial z
    uint16_t* rh = reinterpret_cast<uint16_t*>(smem + Ly::rho_off);
    uint16_t* rl = reinterpret_cast<uint16_t*>(smem + Ly::rho_off + Ly::RHO_BYTES);
    float zp[NT][2];
#pragma unroll
    for (int j = 0; j < NT; ++j) zp[j][0] = zp[j][1] = 0.f;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = warp * 16 + g + half * 8;
      const int tok = tok0 + row;
      const bool vok = row < valid;
      const int pt = tok / (p.Hg * p.W), py = (tok / p.W) % p.Hg, px = tok % p.W;
#pragma unroll
      for (int nj = 0; nj < NT; ++nj) {
        const int col = nj * 8 + 2 * t4;
        const int pr = col >> 1;
        const float p0 = vok ? phi_fast(acc[nj][2 * half]) : 0.f;
        const float p1 = vok ? phi_fast(acc[nj][2 * half + 1]) : 0.f;
        zp[nj][0] += p0;
        zp[nj][1] += p1;
        const int ax = p.rope.axis[pr];
        const int pos = ax == 0 ? pt : (ax == 1 ? py : px);
        const float2 v = M.tab[p.tab_base[pr] + pos * p.tab_stride[pr]];
        const float cs = v.x, sn = v.y;
        const float r0 = p0 * cs - p1 * sn, r1 = p0 * sn + p1 * cs;
        const uint32_t hi = pack_bf16(r0, r1);
        const uint32_t lo = pack_bf16(r0 - bf16_lo(hi), r1 - bf16_hi(hi));
        *reinterpret_cast<uint32_t*>(rh + row * Ly::PS + col) = hi;
        *reinterpret_cast<uint32_t*>(rl + row * Ly::PS + col) = lo;
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
        if (g == 0) M.zpart[warp][nj * 8 + 2 * t4 + e] = x;
      }
    __syncthreads();
    const size_t state = bh * p.nb + blk;
    if (tid < R) {
      float z = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) z += M.zpart[w][tid];
      p.z_blk[state * R + tid] = z;
    }

    // ---- S_j^T pieces: C[r, d] = rho^T V, warp w owns d columns [16w, 16w + 16)
    if (!(ok = __syncthreads_and(mbar_wait(&M.full_v, it & 1, abort)))) break;
    {
      constexpr int MT = R / 16;
      float c2[MT][2][4];
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int e = 0; e < 4; ++e) c2[i][j][e] = 0.f;
      const uint32_t rhb = smem_u32(rh), rlb = smem_u32(rl), vb = smem_u32(sv);
#pragma unroll
      for (int kt = 0; kt < BS; kt += 16) {
        const int arow = kt + (lane & 7) + ((lane >> 4) << 3);
        const int acol = ((lane >> 3) & 1) * 8;
        uint32_t bb[4];
        ldsm_x4_t(bb, vb + sw_off(kt + (lane & 15), warp * 16 + (lane >> 4) * 8));
#pragma unroll
        for (int mi = 0; mi < MT; ++mi) {
          uint32_t ah[4], al[4];
          ldsm_x4_t(ah, rhb + (arow * Ly::PS + mi * 16 + acol) * 2);
          ldsm_x4_t(al, rlb + (arow * Ly::PS + mi * 16 + acol) * 2);
          mma16816(c2[mi][0], ah, bb[0], bb[1]);
          mma16816(c2[mi][0], al, bb[0], bb[1]);
          mma16816(c2[mi][1], ah, bb[2], bb[3]);
          mma16816(c2[mi][1], al, bb[2], bb[3]);
        }
      }
      float* Sout = p.S_blk + state * R * D;
#pragma unroll
      for (int mi = 0; mi < MT; ++mi)
#pragma unroll
        for (int nj = 0; nj < 2; ++nj) {
          const int rr = mi * 16 + g, dd = warp * 16 + nj * 8 + 2 * t4;
          *reinterpret_cast<float2*>(Sout + (size_t)rr * D + dd) = make_float2(c2[mi][nj][0], c2[mi][nj][1]);
          *reinterpret_cast<float2*>(Sout + (size_t)(rr + 8) * D + dd) =
              make_float2(c2[mi][nj][2], c2[mi][nj][3]);
        }
    }
    __syncthreads();  // v is consumed
    if (tid == 0 && it + 1 < my_items) {
      issue_v(it + 1);
      ++v_issued;
    }
  }
  // drain: if we stopped early, let the copies in flight land before exiting
  // (copy i completes phase i of its barrier; items < it were waited for)
  if (tid == 0) {
    int no_abort = 0;
    for (int i = it; i < k_issued; ++i) mbar_wait(&M.full_k, i & 1, &no_abort);
    for (int i = it; i < v_issued; ++i) mbar_wait(&M.full_v, i & 1, &no_abort);
  }
  if (tid == 0 && M.abort && p.dev_err) atomicOr(p.dev_err, ROLA_DEVERR_TIMEOUT);
}

template <int R>
static rola_status_t launch(const rola_shape_t* s, const uint16_t* k, const uint16_t* v, Params prm,
                            cudaStream_t cs) {
  using Ly = Layout<R>;
  CUtensorMap mk, mv;
  if (!rola_host::make_act_map(&mk, k, s, BS) || !rola_host::make_act_map(&mv, v, s, BS))
    return ROLA_ERR_CUDA;
  const size_t smem = Ly::misc_off + sizeof(Misc) + 1024;
  auto kern = rola_prep_kernel<R>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ROLA_ERR_CUDA;
  const int ctas = 2 * rola_host::sm_count();
  const int grid = prm.items < ctas ? prm.items : ctas;
  kern<<<grid, kThreads, smem, cs>>>(mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

}  // namespace prep

// d = 128, 128-token blocks and a latent grid whose rotary table fits in
// shared memory (other shapes take the per-block state kernel and the
// separate pooling pass).
bool prep_kernel_supports(const rola_shape_t* s) {
  if (!(s->d == 128 && s->block == 128 && (s->r == 16 || s->r == 32))) return false;
  const int rh = 2 * (s->r / 6), rt = s->r - 2 * rh;
  const long long entries = (long long)s->T * (rt / 2) + (long long)(s->Hg + s->W) * (rh / 2);
  return entries <= prep::kTabCap;
}

// Block means (if q, qbar and kbar are given) and block states of every
// (batch, head, block); d = 128 and 128-token blocks.
rola_status_t launch_prep_kernel(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const uint16_t* P, double* qbar, double* kbar,
                                 float* S_blk, float* z_blk, int32_t* dev_err, cudaStream_t cs) {
  prep::Params prm{};
  prm.B = s->B;
  prm.H = s->H;
  prm.N = s->N;
  prm.nb = rola_num_blocks(s);
  prm.Hg = s->Hg;
  prm.W = s->W;
  prm.items = s->B * s->H * prm.nb;
  prm.do_pool = (q && qbar && kbar) ? 1 : 0;
  prm.q = q;
  prm.qbar = qbar;
  prm.kbar = kbar;
  prm.P = P;
  prm.S_blk = S_blk;
  prm.z_blk = z_blk;
  prm.dev_err = dev_err;
  rola_host::rope_frequencies(s->r, s->rope_base, prm.rope.freq, prm.rope.axis);
  rola_host::RopeTabLayout tl;
  rola_host::rope_table_layout(s, prm.rope.axis, &tl);
  for (int i = 0; i < 16; ++i) {
    prm.tab_base[i] = tl.base[i];
    prm.tab_stride[i] = tl.stride[i];
  }
  for (int i = 0; i < 17; ++i) prm.tab_first[i] = tl.first[i];
  if (tl.entries > prep::kTabCap) return ROLA_ERR_UNSUPPORTED;
  prm.tab_entries = tl.entries;
  if (s->r == 32) return prep::launch<32>(s, k, v, prm, cs);
  return prep::launch<16>(s, k, v, prm, cs);
}

}  // namespace rola
