// RoLA attention backward on sm_100a (d = 128, 128-token blocks).
//
// The SparkDiffusion write-up (0539edu.com news page, section 05) and the
// project blog ("A simple staging principle", item 1) adapt the dense model to
// 97 % sparsity with a short sparse warm-up, which trains through RoLA: this
// file gives the gradients of the forward of rola_attention_fwd with respect
// to q, k, v, the low-rank projection P_h and the gate, the block mask held
// fixed (selection is a discrete choice).  The pages print no backward; the
// gradient is the chain rule through the forward's steps in reverse:
//   o = o_sp + g o_lin;  o_lin = num / den,  num = rho_q^T S_U,  den = psi_q . z_U
//   dnum = g dO / den,   dden = -g (dO . o_lin) / den,   dg = sum dO . o_lin
//   drho_q = S_U dnum,   dpsi_q = dden z_U + R^T drho_q,   du_q = dpsi_q phi'(u_q)
//   dq += du_q P_h^T,    dP_h += q^T du_q
//   dS_U(a) = rho_q^T dnum, dz_U(a) = sum dden psi_q;  a block state gets the
//   sum over all query blocks minus those that keep it (the mirror of the
//   forward's global-minus-kept complement): dS_b, dz_b
//   dv += rho_k dS_b,  drho_k = dS_b v,  dpsi_k = dz_b + R^T drho_k,  du_k = dpsi_k phi'(u_k)
//   dk += du_k P_h^T,  dP_h += k^T du_k
//   sparse branch: P = exp(S / sqrt(d) - lse), D = dO . o_sp = dO . o - g dO . o_lin,
//   dS = P (dO V^T - D), dq += dS K / sqrt(d), dk += dS^T Q / sqrt(d), dv += P^T dO.
//
// Kernels, in launch order:
//   mask_t_kernel     the transposed block mask: per key block, the ascending
//                     list of query blocks that keep it (integer, exact);
//   bwd_query_kernel  per query block: the query side of the linear branch
//                     (dS_U, dz_U, dq from it, a P_h partial), D per row, and
//                     dq += dS K over the kept blocks -- all contractions on
//                     tcgen05 with accumulators in tensor memory;
//   (states totals)   sum over query blocks of dS_U and dz_U (the forward's
//                     state-totals kernel, float64 sums);
//   bwd_key_kernel    per key block, over the query blocks that keep it:
//                     S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q on
//                     tcgen05, then the key side of the linear branch;
//   bwd_reduce_kernel the P_h and gate partials in a fixed order.
// Nothing is accumulated with atomics: every result is written once, so the
// backward is deterministic.  Linear-branch operands that are not bf16 enter
// the tensor cores as bf16 hi + lo pairs.  Every mbarrier wait is bounded; a
// timeout sets ROLA_DEVERR_TIMEOUT and the CTA drains and returns.
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {
namespace bwd {

constexpr int D = 128, BM = 128, BN = 128;
constexpr uint32_t TILE = BM * D * 2;     // one 128 x 128 bf16 tile, 32 KB
constexpr int kCompute = 128;             // compute threads: thread i owns row (or key) i
constexpr int kThreads = kCompute + 32;   // + one warp: TMA and MMA issue (lane 0)
constexpr int kMaxKept = 256;
constexpr int kMaxBlocks = 1024;

// ---------------------------------------------------------------- operand layouts
// SW128 K-major: `rows` rows of 128-byte atoms, K in atoms of 64 elements
// (the layout the TMA writes for a [rows x 128] bf16 box pair with 128-byte
// swizzle).  The same bytes serve as an MN-major operand with MN = the
// 64-element dimension.
ROLA_DEV uint32_t sw128_off(int row, int k, int rows) {
  return (uint32_t)((k >> 6) * (rows * 128) + row * 128 + ((((k & 63) >> 3) ^ (row & 7)) << 4) + (k & 7) * 2);
}
ROLA_DEV uint64_t desc_kmaj(uint32_t base, int rows, int kk) {
  return smem_desc(base + (uint32_t)(kk >> 2) * rows * 128 + (uint32_t)(kk & 3) * 32, 16, 1024, kSwizzle128B);
}
// MN-major view of a [K rows x 128] SW128 tile (two 64-wide halves `rows` *
// 128 bytes apart), k-step kk covering rows [16 kk, 16 kk + 16).
ROLA_DEV uint64_t desc_mnmaj(uint32_t base, int rows, int kk) {
  return smem_desc(base + (uint32_t)kk * 2048, (uint32_t)rows * 128, 1024, kSwizzle128B);
}
// No-swizzle K-major [rows x KW] operand of 8 x 8 core matrices: element
// (m, k) at (m / 8) * (KW / 8) * 128 + (k / 8) * 128 + (m % 8) * 16 + (k % 8) * 2.
template <int KW>
ROLA_DEV uint32_t core_off(int m, int k) {
  return (uint32_t)((m >> 3) * (KW / 8) * 128 + (k >> 3) * 128 + (m & 7) * 16 + (k & 7) * 2);
}
template <int KW>
ROLA_DEV uint64_t desc_core(uint32_t base, int kk) {
  return smem_desc(base + (uint32_t)kk * 256, 128, (KW / 8) * 128, kSwizzleNone);
}

ROLA_DEV void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
  const uint32_t h = f2bf(x);
  hi = (uint16_t)h;
  lo = (uint16_t)f2bf(x - __uint_as_float(h << 16));
}

// 3-D rotary pair of a token (t, y, x); pair pr turns by pos(axis) * freq.
constexpr int kTabCap = 1024;  // cos/sin entries of the rotary table in shared memory

struct Params {
  int B, H, N, nb, kb, T, Hg, W;
  float scale;       // 1 / sqrt(d)
  float scale_log2;  // log2(e) / sqrt(d)
  int chunk;         // blocks per CTA (query blocks, or key blocks)
  const uint16_t* P;
  const float* gate;
  const int32_t* idx;
  const float* S_blk;
  const float* z_blk;
  const float* S_glb;
  const float* z_glb;
  const uint16_t* out;
  const uint16_t* out_lo;
  const uint16_t* dout;
  const float* lse;
  const float* den;
  const int32_t* mt_off;   // [B, H, nb + 1]
  const int32_t* mt_rows;  // [B, H, nb * kb]
  float* dSU;              // [B, H, nb, r, d]
  float* dzU;              // [B, H, nb, r]
  const float* dSU_tot;    // [B, H, r, d]
  const float* dzU_tot;    // [B, H, r]
  float* Drow;             // [B, H, N]
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  float* dP_part;          // [B, H, chunks_q + chunks_k, d, r]
  float* dg_part;          // [B, H, chunks_q]
  int chunks_q, chunks_k;
  int32_t* dev_err;
  RopeTable rope;
  // rotary table: entry of pair pr at position pos = tab_base[pr] + pos * tab_stride[pr];
  // pair pr fills entries [tab_first[pr], tab_first[pr + 1]) of the fill order
  int tab_base[16], tab_stride[16], tab_first[17];
  int tab_entries;
};

// (cos, sin) of rotation pair pr at the row's grid position, from the table
ROLA_DEV void rope_cs(const Params& p, const float2* tab, int pr, int pt, int py, int px, float& c, float& s) {
  const int ax = p.rope.axis[pr];
  const float2 v = tab[p.tab_base[pr] + (ax == 0 ? pt : (ax == 1 ? py : px)) * p.tab_stride[pr]];
  c = v.x;
  s = v.y;
}
// The table, once per CTA: the same rope_sincos values the forward's table holds.
ROLA_DEV void fill_rope_table(const Params& p, float2* tab, int R, int nthreads) {
  for (int e = (int)threadIdx.x; e < p.tab_entries; e += nthreads) {
    int pr = 0;
    while (pr + 1 < R / 2 && e >= p.tab_first[pr + 1]) ++pr;
    const int pos = e - p.tab_first[pr];
    float sn, cs;
    rope_sincos(pos, p.rope.freq[pr], &sn, &cs);
    tab[p.tab_base[pr] + pos * p.tab_stride[pr]] = make_float2(cs, sn);
  }
}

// ================================================================ transposed mask
// One CTA per (b, h): bits[j][w] bit (a & 31) of word a >> 5 is set when query
// block a keeps key block j; a key block's list is its set bits in ascending
// order.  Entries out of range or not ascending are skipped (as the forward
// skips them) and reported.
__global__ void __launch_bounds__(512) mask_t_kernel(const int32_t* __restrict__ idx, int nb, int kb,
                                                     int32_t* __restrict__ off_out, int32_t* __restrict__ rows_out,
                                                     int32_t* dev_err) {
  extern __shared__ uint32_t mt_sm[];
  const int words = (nb + 31) >> 5;
  uint32_t* bits = mt_sm;                                              // [nb][words]
  int32_t* off = reinterpret_cast<int32_t*>(mt_sm + (size_t)nb * words);  // [nb + 1]
  const size_t bh = blockIdx.x;
  const int32_t* id = idx + bh * (size_t)nb * kb;
  for (int e = threadIdx.x; e < nb * words; e += blockDim.x) bits[e] = 0u;
  __syncthreads();
  int bad = 0;
  for (int e = threadIdx.x; e < nb * kb; e += blockDim.x) {
    const int a = e / kb, i = e % kb, j = id[e];
    if (j < 0 || j >= nb || (i > 0 && j <= id[e - 1])) {
      bad = 1;
      continue;
    }
    atomicOr(&bits[j * words + (a >> 5)], 1u << (a & 31));
  }
  if (bad && dev_err) atomicOr(dev_err, ROLA_DEVERR_BAD_INDEX);
  __syncthreads();
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    int c = 0;
    for (int w = 0; w < words; ++w) c += __popc(bits[j * words + w]);
    off[j + 1] = c;
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // n_blocks <= 1024: a serial scan takes a few microseconds
    off[0] = 0;
    for (int j = 0; j < nb; ++j) off[j + 1] += off[j];
  }
  __syncthreads();
  int32_t* ro = rows_out + bh * (size_t)nb * kb;
  for (int j = threadIdx.x; j <= nb; j += blockDim.x) off_out[bh * (nb + 1) + j] = off[j];
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    int pos = off[j];
    for (int w = 0; w < words; ++w)
      for (uint32_t m = bits[j * words + w]; m; m &= m - 1) ro[pos++] = w * 32 + __ffs(m) - 1;
  }
}

// ================================================================ shared pieces

// Bounded wait of the whole warp; false on a timeout or an abort elsewhere.
ROLA_DEV bool wwait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const bool ok = mbar_wait(bar, parity, abort);
  return __all_sync(0xffffffffu, ok);
}

// The kept list of query block a, validated as the forward validates it
// (in range, strictly ascending); returns the number of valid entries written
// to `list` and sets *bad when an entry was skipped.
ROLA_DEV int kept_list(const int32_t* row, int kb, int nb, int* list, int* bad) {
  int n = 0;
  for (int e = 0; e < kb; ++e) {
    const int v = row[e];
    if (v < 0 || v >= nb || (e > 0 && v <= row[e - 1])) {
      *bad = 1;
      continue;
    }
    list[n++] = v;
  }
  return n;
}

// Token coordinates on the (T, Hg, W) grid.
ROLA_DEV void coords(int n, int Hg, int W, int& t, int& y, int& x) {
  const int hw = Hg * W;
  t = n / hw;
  const int rem = n - t * hw;
  y = rem / W;
  x = rem - y * W;
}

template <int R>
struct QLayout {
  static constexpr uint32_t q_off = 0, do_off = TILE;
  static constexpr uint32_t ring_off = 2 * TILE;                  // 2 stages x (K, V)
  static constexpr uint32_t pt_off = ring_off + 4 * TILE;         // P_h^T, SW128 K-major [r x d]
  static constexpr uint32_t pc_off = pt_off + R * D * 2;          // P_h, core K-major [d x r]
  static constexpr uint32_t misc_off = pc_off + R * D * 2;
  // scratch of the linear phase, inside the (then idle) ring
  static constexpr uint32_t su_off = ring_off;                    // S_U hi, lo: SW128 [r x d]
  static constexpr uint32_t rho_off = su_off + 2 * R * D * 2;     // rho hi, lo: core [128 x r]
  static constexpr uint32_t rht_off = rho_off + 2 * BM * R * 2;   // (c rho)^T hi, lo: SW128 [r x 128]
  static constexpr uint32_t du_off = rht_off + 2 * R * BM * 2;    // du hi, lo: core [128 x r]
  static constexpr uint32_t dut_off = du_off + 2 * BM * R * 2;    // du^T hi, lo: SW128 [r x 128]
  static_assert(dut_off + 2 * R * BM * 2 <= ring_off + 4 * TILE, "linear scratch must fit the ring");
  static_assert((R * D * 2) % 1024 == 0 && (BM * R * 2) % 1024 == 0, "1024-byte aligned operands");
};

struct QMisc {
  uint64_t load, mma, s_ready, p_ready, full[2], empty[2], d_ready;
  uint32_t tmem;
  int abort;
  int err;
  int nk;
  int lin_empty;
  int list[kMaxKept];
  float zU[32];
  float red[4][32];
  float lse2[BM];
  float Dr[BM];
  float2 tab[kTabCap];
};

// TMEM columns of the query-major kernel
constexpr uint32_t kQ_dq = 0, kQ_S = 128, kQ_dP = 256, kQ_uq = 384, kQ_ds = 416, kQ_dsu = 448, kQ_dph = 480;
constexpr uint32_t kQ_S2 = 384;  // the sparse loop's second S buffer (over the linear phase's columns)

// ================================================================ query-major pass
template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_query_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const Params p) {
  using L = QLayout<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  QMisc& M = *reinterpret_cast<QMisc*>(smem + L::misc_off);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * p.H + h;
  const bool issuer = tid == kCompute;
  volatile int* abort = &M.abort;
  // A CTA that already timed out in this launch makes the rest skip their work.
  if (__syncthreads_or(tid == 0 && p.dev_err &&
                       (*reinterpret_cast<volatile int32_t*>(p.dev_err) & ROLA_DEVERR_TIMEOUT)))
    return;

  if (tid == 0) {
    mbar_init(&M.load, 1);
    mbar_init(&M.mma, 1);
    mbar_init(&M.s_ready, 1);
    mbar_init(&M.p_ready, kCompute);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&M.full[i], 1);
      mbar_init(&M.empty[i], 1);
    }
    mbar_init(&M.d_ready, 1);
    M.abort = 0;
    M.err = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&M.tmem, 512);
    tmem_relinquish();
  }
  fill_rope_table(p, M.tab, R, kThreads);
  // P_h operands of this head: P_h^T (SW128 K-major, N = r rows, K = d) and
  // P_h (core K-major, N = d rows, K = r); P_h is bf16, so no lo part
  for (int e = tid; e < D * R; e += kThreads) {
    const int c = e / R, rr = e % R;  // P_h[c][rr]
    const uint16_t w = p.P[((size_t)h * D + c) * R + rr];
    *reinterpret_cast<uint16_t*>(smem + L::pt_off + sw128_off(rr, c, R)) = w;
    *reinterpret_cast<uint16_t*>(smem + L::pc_off + core_off<R>(c, rr)) = w;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = M.tmem;
  const uint32_t trow = tm + ((uint32_t)((warp & 3) * 32) << 16);  // this warp's lane quarter
  const float g = p.gate[h];
  // phase counters of the barriers; ce counts the commits to empty[] (a
  // stage's commits outnumber the waits on it, so its parity follows the commits)
  uint32_t ph_load = 0, ph_mma = 0, ph_s = 0, ph_p = 0, ph_full[2] = {0, 0}, ce[2] = {0, 0}, ph_d = 0;
  float dph[R];  // thread t (< 128) accumulates row t (= d index) of this CTA's P_h partial
#pragma unroll
  for (int i = 0; i < R; ++i) dph[i] = 0.f;
  float dg_acc = 0.f;
  bool ok = true;
  const int a0 = chunk * p.chunk;

  for (int a = a0; ok && a < min(a0 + p.chunk, p.nb); ++a) {
    // ---- kept list, loads of Q_a and dO_a
    if (tid == 0) {
      int bad = 0;
      M.nk = kept_list(p.idx + (bh * p.nb + a) * p.kb, p.kb, p.nb, M.list, &bad);
      M.lin_empty = M.nk >= p.nb;
      if (bad) M.err = 1;
    }
    if (issuer) {
      mbar_expect_tx(&M.load, 2 * TILE);
      for (int ka = 0; ka < 2; ++ka) {
        tma_load_4d(smem + L::q_off + ka * (BM * 128), &tmQ, &M.load, ka * 64, h, a * BM, b);
        tma_load_4d(smem + L::do_off + ka * (BM * 128), &tmO, &M.load, ka * 64, h, a * BM, b);
      }
    }
    __syncthreads();
    const int nk = M.nk;
    const bool lin = !M.lin_empty;
    // ---- per-row statistics and the complement state S_U, z_U
    const int n = a * BM + tid;
    const bool valid = tid < kCompute && n < p.N;
    float lse2 = INFINITY, c_row = 0.f, den = 1.f, Dfull = 0.f;
    int pt = 0, py = 0, px = 0;
    if (tid < kCompute) {
      // D's first term dO . o, from the output and its bf16 rounding residual
      // (the rounding of o alone would cost D ~2^-9 of |dO| |o|).  A warp
      // reads its 32 rows two at a time, 16 lanes x 16 bytes per row of each
      // of out, out_lo and dout (coalesced), and sums each row over its 16
      // lanes; row i's sum lands in M.Dr[i] for its owner thread.
      {
        const int half = lane >> 4, l16 = lane & 15;
#pragma unroll 4
        for (int i2 = 0; i2 < 16; ++i2) {
          const int r = warp * 32 + 2 * i2 + half, nr = a * BM + r;
          float part = 0.f;
          if (nr < p.N) {
            const size_t ao = ((b * (size_t)p.N + nr) * p.H + h) * D + l16 * 8;
            const uint4 o4 = __ldg(reinterpret_cast<const uint4*>(p.out + ao));
            const uint4 l4 = __ldg(reinterpret_cast<const uint4*>(p.out_lo + ao));
            const uint4 d4 = __ldg(reinterpret_cast<const uint4*>(p.dout + ao));
            const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w}, lw[4] = {l4.x, l4.y, l4.z, l4.w};
            const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              part += (bf16_lo(ow[i]) + bf16_lo(lw[i])) * bf16_lo(dw[i]) +
                      (bf16_hi(ow[i]) + bf16_hi(lw[i])) * bf16_hi(dw[i]);
          }
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          if (l16 == 0) M.Dr[r] = part;
        }
        __syncwarp();
      }
      if (valid) {
        const size_t ro = bh * p.N + n;
        lse2 = p.lse[ro] * 1.4426950408889634f;
        den = p.den[ro];
        c_row = lin ? g / den : 0.f;
        Dfull = M.Dr[tid];
        coords(n, p.Hg, p.W, pt, py, px);
      }
      // S_U column d = tid: S - sum over the kept blocks (fp32, as the forward)
      float su[R];
      const float* Sg = p.S_glb + bh * R * D;
#pragma unroll
      for (int r = 0; r < R; ++r) su[r] = Sg[r * D + tid];
      float zu = tid < R ? p.z_glb[bh * R + tid] : 0.f;
      // four blocks' loads in flight per round trip; the subtractions keep
      // the kept list's order
      int e = 0;
      for (; e + 4 <= nk; e += 4) {
        float t[4][R];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float* Sb = p.S_blk + (bh * p.nb + M.list[e + i]) * R * D;
#pragma unroll
          for (int r = 0; r < R; ++r) t[i][r] = __ldg(Sb + r * D + tid);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int r = 0; r < R; ++r) su[r] -= t[i][r];
        if (tid < R)
          for (int i = 0; i < 4; ++i) zu -= p.z_blk[(bh * p.nb + M.list[e + i]) * R + tid];
      }
      for (; e < nk; ++e) {
        const size_t st = bh * p.nb + M.list[e];
        const float* Sb = p.S_blk + st * R * D;
#pragma unroll
        for (int r = 0; r < R; ++r) su[r] -= Sb[r * D + tid];
        if (tid < R) zu -= p.z_blk[st * R + tid];
      }
      if (tid < R) M.zU[tid] = zu;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint16_t hi, lo;
        split_bf16(su[r], hi, lo);
        *reinterpret_cast<uint16_t*>(smem + L::su_off + sw128_off(r, tid, R)) = hi;
        *reinterpret_cast<uint16_t*>(smem + L::su_off + R * D * 2 + sw128_off(r, tid, R)) = lo;
      }
      M.lse2[tid] = lse2;
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- u_q = Q P_h
    constexpr uint32_t id_qr = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, R);
    constexpr uint32_t id_ol = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, D);
    constexpr uint32_t id_tr = instr_desc(kFmtBF16, kFmtBF16, true, false, 128, R);
    constexpr uint32_t id_dd = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, D);
    constexpr uint32_t id_pv = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, BN);
    const uint32_t sQ = smem_u32(smem + L::q_off), sO = smem_u32(smem + L::do_off);
    const uint32_t sPT = smem_u32(smem + L::pt_off), sPC = smem_u32(smem + L::pc_off);
    const uint32_t sSU = smem_u32(smem + L::su_off), sRho = smem_u32(smem + L::rho_off);
    const uint32_t sRht = smem_u32(smem + L::rht_off), sDu = smem_u32(smem + L::du_off);
    const uint32_t sDut = smem_u32(smem + L::dut_off);
    if (issuer) {
      ok = mbar_wait(&M.load, ph_load & 1, abort);
      if (ok) {
        tc_fence_after();
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + kQ_uq, desc_kmaj(sQ, BM, kk), desc_kmaj(sPT, R, kk), id_qr, kk > 0);
      }
      mma_commit(&M.mma);
    }
    ++ph_load;
    float u[R], psi[R];
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort);
      tc_fence_after();
      uint32_t v[32];
      if (R == 32) tmem_ld32(trow + kQ_uq, v);
      else tmem_ld16(trow + kQ_uq, *reinterpret_cast<uint32_t(*)[16]>(v));
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < R; ++i) {
        u[i] = valid ? __uint_as_float(v[i]) : 0.f;
        psi[i] = phi_fast(u[i]);
      }
      // rho (core K-major A) and (c rho)^T (SW128 K-major B over the rows)
#pragma unroll
      for (int pr = 0; pr < R / 2; ++pr) {
        float cs, sn;
        rope_cs(p, M.tab, pr, pt, py, px, cs, sn);
        const float r0 = psi[2 * pr] * cs - psi[2 * pr + 1] * sn;
        const float r1 = psi[2 * pr] * sn + psi[2 * pr + 1] * cs;
        uint16_t h0, l0, h1, l1;
        split_bf16(r0, h0, l0);
        split_bf16(r1, h1, l1);
        const uint32_t off = core_off<R>(tid, 2 * pr);
        *reinterpret_cast<uint32_t*>(smem + L::rho_off + off) = h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t*>(smem + L::rho_off + BM * R * 2 + off) = l0 | ((uint32_t)l1 << 16);
        split_bf16(c_row * r0, h0, l0);
        split_bf16(c_row * r1, h1, l1);
        *reinterpret_cast<uint16_t*>(smem + L::rht_off + sw128_off(2 * pr, tid, R)) = h0;
        *reinterpret_cast<uint16_t*>(smem + L::rht_off + sw128_off(2 * pr + 1, tid, R)) = h1;
        *reinterpret_cast<uint16_t*>(smem + L::rht_off + R * BM * 2 + sw128_off(2 * pr, tid, R)) = l0;
        *reinterpret_cast<uint16_t*>(smem + L::rht_off + R * BM * 2 + sw128_off(2 * pr + 1, tid, R)) = l1;
      }
    }
    ++ph_mma;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- o_lin * den = rho S_U,  dO S_U^T,  dS_U^T = dO^T (c rho)
    if (issuer && ok) {
      tc_fence_after();
      for (int kk = 0; kk < R / 16; ++kk) {
        const uint64_t ah = desc_core<R>(sRho, kk), al = desc_core<R>(sRho + BM * R * 2, kk);
        const uint64_t bh_ = desc_mnmaj(sSU, R, kk), bl_ = desc_mnmaj(sSU + R * D * 2, R, kk);
        mma_ss(tm + kQ_S, ah, bh_, id_ol, kk > 0);
        mma_ss(tm + kQ_S, ah, bl_, id_ol, 1);
        mma_ss(tm + kQ_S, al, bh_, id_ol, 1);
      }
      for (int kk = 0; kk < D / 16; ++kk) {
        mma_ss(tm + kQ_ds, desc_kmaj(sO, BM, kk), desc_kmaj(sSU, R, kk), id_qr, kk > 0);
        mma_ss(tm + kQ_ds, desc_kmaj(sO, BM, kk), desc_kmaj(sSU + R * D * 2, R, kk), id_qr, 1);
      }
      for (int kk = 0; kk < BM / 16; ++kk) {
        mma_ss(tm + kQ_dsu, desc_mnmaj(sO, BM, kk), desc_kmaj(sRht, R, kk), id_tr, kk > 0);
        mma_ss(tm + kQ_dsu, desc_mnmaj(sO, BM, kk), desc_kmaj(sRht + R * BM * 2, R, kk), id_tr, 1);
      }
    }
    if (issuer) mma_commit(&M.mma);
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort) && ok;
      tc_fence_after();
      // o_lin . dO and D
      float old = 0.f;
      const uint4* drow = reinterpret_cast<const uint4*>(p.dout + ((b * (size_t)p.N + (valid ? n : 0)) * p.H + h) * D);
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kQ_S + c * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int e8 = 0; e8 < 4; ++e8) {
          const uint4 d4 = valid ? __ldg(drow + c * 4 + e8) : make_uint4(0, 0, 0, 0);
          const uint32_t dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int q2 = 0; q2 < 4; ++q2)
            old += __uint_as_float(v[e8 * 8 + 2 * q2]) * bf16_lo(dw[q2]) +
                   __uint_as_float(v[e8 * 8 + 2 * q2 + 1]) * bf16_hi(dw[q2]);
        }
      }
      old = lin && valid ? old / den : 0.f;  // dO . o_lin
      const float Dv = valid ? Dfull - g * old : 0.f;
      M.Dr[tid] = Dv;
      if (valid) p.Drow[bh * p.N + n] = Dv;
      dg_acc += old;
      const float dden = lin && valid ? -g * old / den : 0.f;
      // dpsi = dden z_U + R^T (c dO S_U^T), du = dpsi phi'(u)
      uint32_t w[32];
      if (R == 32) tmem_ld32(trow + kQ_ds, w);
      else tmem_ld16(trow + kQ_ds, *reinterpret_cast<uint32_t(*)[16]>(w));
      tmem_wait_ld();
#pragma unroll
      for (int pr = 0; pr < R / 2; ++pr) {
        float cs, sn;
        rope_cs(p, M.tab, pr, pt, py, px, cs, sn);
        const float d0 = c_row * __uint_as_float(w[2 * pr]), d1 = c_row * __uint_as_float(w[2 * pr + 1]);
        // R^T of the pair rotation: (d0 cs + d1 sn, -d0 sn + d1 cs)
        const float p0 = dden * M.zU[2 * pr] + d0 * cs + d1 * sn;
        const float p1 = dden * M.zU[2 * pr + 1] - d0 * sn + d1 * cs;
        const float du0 = valid ? p0 * (u[2 * pr] > 0.f ? 1.f : psi[2 * pr]) : 0.f;
        const float du1 = valid ? p1 * (u[2 * pr + 1] > 0.f ? 1.f : psi[2 * pr + 1]) : 0.f;
        uint16_t h0, l0, h1, l1;
        split_bf16(du0, h0, l0);
        split_bf16(du1, h1, l1);
        const uint32_t off = core_off<R>(tid, 2 * pr);
        *reinterpret_cast<uint32_t*>(smem + L::du_off + off) = h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t*>(smem + L::du_off + BM * R * 2 + off) = l0 | ((uint32_t)l1 << 16);
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + sw128_off(2 * pr, tid, R)) = h0;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + sw128_off(2 * pr + 1, tid, R)) = h1;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + R * BM * 2 + sw128_off(2 * pr, tid, R)) = l0;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + R * BM * 2 + sw128_off(2 * pr + 1, tid, R)) = l1;
      }
      // dz_U(a) = sum over rows of dden psi (fixed-order reduction)
#pragma unroll
      for (int i = 0; i < R; ++i) {
        float x = dden * psi[i];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) M.red[warp][i] = x;
      }
      // dS_U(a) from dS_U^T in tensor memory: thread t holds column d = t
      uint32_t t32[32];
      if (R == 32) tmem_ld32(trow + kQ_dsu, t32);
      else tmem_ld16(trow + kQ_dsu, *reinterpret_cast<uint32_t(*)[16]>(t32));
      tmem_wait_ld();
      float* dsu = p.dSU + (bh * p.nb + a) * R * D;
#pragma unroll
      for (int r = 0; r < R; ++r) dsu[r * D + tid] = lin ? __uint_as_float(t32[r]) : 0.f;
    }
    ++ph_mma;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid < R) p.dzU[(bh * p.nb + a) * R + tid] = M.red[0][tid] + M.red[1][tid] + M.red[2][tid] + M.red[3][tid];
    // ---- dq = du P_h^T (starts the dq accumulator), P_h partial = Q^T du
    if (issuer && ok) {
      tc_fence_after();
      for (int kk = 0; kk < R / 16; ++kk) {
        mma_ss(tm + kQ_dq, desc_core<R>(sDu, kk), desc_core<R>(sPC, kk), id_dd, kk > 0);
        mma_ss(tm + kQ_dq, desc_core<R>(sDu + BM * R * 2, kk), desc_core<R>(sPC, kk), id_dd, 1);
      }
      for (int kk = 0; kk < BM / 16; ++kk) {
        mma_ss(tm + kQ_dph, desc_mnmaj(sQ, BM, kk), desc_kmaj(sDut, R, kk), id_tr, kk > 0);
        mma_ss(tm + kQ_dph, desc_mnmaj(sQ, BM, kk), desc_kmaj(sDut + R * BM * 2, R, kk), id_tr, 1);
      }
    }
    if (issuer) mma_commit(&M.mma);
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort) && ok;
      tc_fence_after();
      uint32_t t32[32];
      if (R == 32) tmem_ld32(trow + kQ_dph, t32);
      else tmem_ld16(trow + kQ_dph, *reinterpret_cast<uint32_t(*)[16]>(t32));
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < R; ++i) dph[i] += __uint_as_float(t32[i]);
    }
    ++ph_mma;
    tc_fence_before();
    __syncthreads();  // the linear scratch (ring) is free again
    // ---- sparse branch: per kept block S = Q K^T, dP = dO V^T, dS, dq += dS K
    if (issuer && ok) {
      auto load_kv = [&](int t) {
        const int st = t & 1, blk = M.list[t];
        mbar_expect_tx(&M.full[st], 2 * TILE);
        for (int ka = 0; ka < 2; ++ka) {
          tma_load_4d(smem + L::ring_off + (2 * st) * TILE + ka * (BN * 128), &tmK, &M.full[st], ka * 64, h,
                      blk * BN, b);
          tma_load_4d(smem + L::ring_off + (2 * st + 1) * TILE + ka * (BN * 128), &tmV, &M.full[st], ka * 64, h,
                      blk * BN, b);
        }
      };
      // S of pair t goes to one of two buffers (columns 128 and 384; the
      // latter hold the linear phase's operands, done by now), dP to one
      auto sbuf = [](int t) -> uint32_t { return (t & 1) ? kQ_S2 : kQ_S; };
      auto issue_S = [&](int t) -> bool {
        const int st = t & 1;
        if (!mbar_wait(&M.full[st], ph_full[st] & 1, abort)) return false;
        ++ph_full[st];
        tc_fence_after();
        const uint32_t sK = smem_u32(smem + L::ring_off + (2 * st) * TILE);
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + sbuf(t), desc_kmaj(sQ, BM, kk), desc_kmaj(sK, BN, kk), id_dd, kk > 0);
        mma_commit(&M.s_ready);
        return true;
      };
      auto issue_dP = [&](int t) {
        const uint32_t sV = smem_u32(smem + L::ring_off + (2 * (t & 1) + 1) * TILE);
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + kQ_dP, desc_kmaj(sO, BM, kk), desc_kmaj(sV, BN, kk), id_dd, kk > 0);
        mma_commit(&M.d_ready);
      };
      for (int t = 0; t < min(nk, 2); ++t) load_kv(t);
      if (nk > 0 && (ok = issue_S(0))) issue_dP(0);
      // per pair t: S(t + 1) first (the next pair's exponentials need only
      // it), then dq += dS(t) K(t), then dP(t + 1) (it overwrites the dP
      // columns, which hold dS(t)'s lo part until that MMA has read them)
      for (int t = 0; ok && t < nk; ++t) {
        const int st = t & 1;
        if (!(ok = mbar_wait(&M.p_ready, ph_p & 1, abort))) break;
        ++ph_p;
        tc_fence_after();
        if (t + 1 < nk && !(ok = issue_S(t + 1))) break;
        const uint32_t sK = smem_u32(smem + L::ring_off + (2 * st) * TILE);
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ts(tm + kQ_dq, tm + sbuf(t) + kk * 8, desc_mnmaj(sK, BN, kk), id_pv, 1);
          mma_ts(tm + kQ_dq, tm + kQ_dP + kk * 8, desc_mnmaj(sK, BN, kk), id_pv, 1);
        }
        mma_commit(&M.empty[st]);
        const uint32_t my = ce[st]++;
        if (t + 1 < nk) issue_dP(t + 1);
        if (t + 2 < nk) {
          if (!(ok = mbar_wait(&M.empty[st], my & 1, abort))) break;
          load_kv(t + 2);
        }
      }
      mma_commit(&M.mma);
    } else if (issuer) {
      mma_commit(&M.mma);
    }
    if (tid < kCompute) {
      const float Dv = M.Dr[tid];
      for (int t = 0; ok && t < nk; ++t) {
        const uint32_t sb = (t & 1) ? kQ_S2 : kQ_S;
        if (!(ok = wwait(&M.s_ready, ph_s & 1, abort))) break;
        ++ph_s;
        tc_fence_after();
        const int blk = M.list[t];
        const int kvalid = min(BN, p.N - blk * BN);
        // phase 1 (while dq += dS(t - 1) K and dP run): P in fp32 over S
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t sv[32];
          tmem_ld32(trow + sb + c * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c0 = c * 32 + e;
            sv[e] = __float_as_uint(c0 < kvalid ? fast_exp2(__uint_as_float(sv[e]) * p.scale_log2 - lse2) : 0.f);
          }
          tmem_st32(trow + sb + c * 32, sv);
        }
        tmem_wait_st();
        if (!(ok = wwait(&M.d_ready, ph_d & 1, abort))) break;
        ++ph_d;
        tc_fence_after();
        // phase 2: dS as bf16 hi (over the read P columns) + lo (over the read
        // dP columns): dq sums dS K over the kept keys with cancellation, where
        // the bf16 rounding of dS alone is ~2^-9 of sum |dS K|
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t sv[32], dv[32], pk[16], pl[16];
          tmem_ld32(trow + sb + c * 32, sv);
          tmem_ld32(trow + kQ_dP + c * 32, dv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = __uint_as_float(sv[2 * e]), p1 = __uint_as_float(sv[2 * e + 1]);
            const float d0 = p0 * (__uint_as_float(dv[2 * e]) - Dv) * p.scale;
            const float d1 = p1 * (__uint_as_float(dv[2 * e + 1]) - Dv) * p.scale;
            pk[e] = pack_bf16(d0, d1);
            pl[e] = pack_bf16(d0 - bf16_lo(pk[e]), d1 - bf16_hi(pk[e]));
          }
          tmem_st16(trow + sb + c * 16, pk);
          tmem_st16(trow + kQ_dP + c * 16, pl);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&M.p_ready);
      }
      if (ok) ok = wwait(&M.mma, ph_mma & 1, abort);
      tc_fence_after();
      // dq row (padding rows are not written)
      uint16_t* dst = p.dq + ((b * (size_t)p.N + (valid ? n : 0)) * p.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(trow + kQ_dq + c * 32, v);
        tmem_wait_ld();
        if (valid && ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            d4[q4] = make_uint4(pack_bf16(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
        }
      }
    }
    ++ph_mma;
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
  }
  // ---- partials of P_h (row d = tid) and of the gate
  if (tid < kCompute) {
    float* dst = p.dP_part + ((bh * (p.chunks_q + p.chunks_k)) + chunk) * D * R + tid * R;
#pragma unroll
    for (int i = 0; i < R; ++i) dst[i] = dph[i];
    float x = dg_acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) M.red[warp][0] = x;
  }
  __syncthreads();
  if (tid == 0) p.dg_part[bh * p.chunks_q + chunk] = M.red[0][0] + M.red[1][0] + M.red[2][0] + M.red[3][0];
  // teardown: every issued MMA has completed (each phase waited on its commit)
  if (issuer) {
    mma_commit(&M.mma);
    int no_abort = 0;
    mbar_wait(&M.mma, ph_mma & 1, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  if (tid == 0 && p.dev_err && (M.abort || M.err))
    atomicOr(p.dev_err, (M.abort ? ROLA_DEVERR_TIMEOUT : 0) | (M.err ? ROLA_DEVERR_BAD_INDEX : 0));
}

// ================================================================ key-major pass
template <int R>
struct KLayout {
  static constexpr uint32_t k_off = 0, v_off = TILE;
  static constexpr uint32_t ring_off = 2 * TILE;                  // 2 stages x (Q_a, dO_a)
  static constexpr uint32_t pt_off = ring_off + 4 * TILE;         // P_h^T, SW128 K-major [r x d]
  static constexpr uint32_t pc_off = pt_off + R * D * 2;          // P_h, core K-major [d x r]
  static constexpr uint32_t misc_off = pc_off + R * D * 2;
  // scratch of the linear phase, inside the (then idle) ring
  static constexpr uint32_t sb_off = ring_off;                    // dS_b hi, lo: SW128 [r x d]
  static constexpr uint32_t rho_off = sb_off + 2 * R * D * 2;     // rho_k hi, lo: core [128 x r]
  static constexpr uint32_t du_off = rho_off + 2 * BN * R * 2;    // du hi, lo: core [128 x r]
  static constexpr uint32_t dut_off = du_off + 2 * BN * R * 2;    // du^T hi, lo: SW128 [r x 128]
  static_assert(dut_off + 2 * R * BN * 2 <= ring_off + 4 * TILE, "linear scratch must fit the ring");
};

struct KMisc {
  uint64_t load, mma, s_ready, p_ready, full[2], empty[2], d_ready;
  uint32_t tmem;
  int abort;
  int nkeep;
  int keep[kMaxBlocks];
  float zb[32];
  float lse2[2][BM];
  float Dr[2][BM];
  float2 tab[kTabCap];
};

// TMEM columns of the key-major kernel
constexpr uint32_t kK_S = 0, kK_dP = 128, kK_dV = 256, kK_dK = 384;

template <int R>
__global__ void __launch_bounds__(kThreads, 1)
    bwd_key_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                   const Params p) {
  using L = KLayout<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KMisc& M = *reinterpret_cast<KMisc*>(smem + L::misc_off);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int chunk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = (size_t)b * p.H + h;
  const bool issuer = tid == kCompute;
  volatile int* abort = &M.abort;
  if (__syncthreads_or(tid == 0 && p.dev_err &&
                       (*reinterpret_cast<volatile int32_t*>(p.dev_err) & ROLA_DEVERR_TIMEOUT)))
    return;

  if (tid == 0) {
    mbar_init(&M.load, 1);
    mbar_init(&M.mma, 1);
    mbar_init(&M.s_ready, 1);
    mbar_init(&M.p_ready, kCompute);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&M.full[i], 1);
      mbar_init(&M.empty[i], 1);
    }
    mbar_init(&M.d_ready, 1);
    M.abort = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&M.tmem, 512);
    tmem_relinquish();
  }
  fill_rope_table(p, M.tab, R, kThreads);
  for (int e = tid; e < D * R; e += kThreads) {
    const int c = e / R, rr = e % R;
    const uint16_t w = p.P[((size_t)h * D + c) * R + rr];
    *reinterpret_cast<uint16_t*>(smem + L::pt_off + sw128_off(rr, c, R)) = w;
    *reinterpret_cast<uint16_t*>(smem + L::pc_off + core_off<R>(c, rr)) = w;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = M.tmem;
  const uint32_t trow = tm + ((uint32_t)((warp & 3) * 32) << 16);
  uint32_t ph_load = 0, ph_mma = 0, ph_s = 0, ph_p = 0, ph_full[2] = {0, 0}, ce[2] = {0, 0}, ph_d = 0;
  float dph[R];
#pragma unroll
  for (int i = 0; i < R; ++i) dph[i] = 0.f;
  bool ok = true;
  constexpr uint32_t id_dd = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, D);
  constexpr uint32_t id_pv = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, D);
  constexpr uint32_t id_qr = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, R);
  constexpr uint32_t id_tr = instr_desc(kFmtBF16, kFmtBF16, true, false, 128, R);
  const uint32_t sK = smem_u32(smem + L::k_off), sV = smem_u32(smem + L::v_off);
  const uint32_t sPT = smem_u32(smem + L::pt_off), sPC = smem_u32(smem + L::pc_off);
  const uint32_t sSb = smem_u32(smem + L::sb_off), sRho = smem_u32(smem + L::rho_off);
  const uint32_t sDu = smem_u32(smem + L::du_off), sDut = smem_u32(smem + L::dut_off);
  const int j0 = chunk * p.chunk;

  for (int j = j0; ok && j < min(j0 + p.chunk, p.nb); ++j) {
    if (tid == 0) {
      const int32_t* off = p.mt_off + bh * (p.nb + 1);
      const int o0 = off[j], o1 = off[j + 1];
      M.nkeep = o1 - o0;
      for (int e = 0; e < o1 - o0; ++e) M.keep[e] = p.mt_rows[bh * (size_t)p.nb * p.kb + o0 + e];
    }
    if (issuer) {
      mbar_expect_tx(&M.load, 2 * TILE);
      for (int ka = 0; ka < 2; ++ka) {
        tma_load_4d(smem + L::k_off + ka * (BN * 128), &tmK, &M.load, ka * 64, h, j * BN, b);
        tma_load_4d(smem + L::v_off + ka * (BN * 128), &tmV, &M.load, ka * 64, h, j * BN, b);
      }
    }
    __syncthreads();
    const int nkeep = M.nkeep;
    const int key = j * BN + tid;
    const bool kvalid = tid < kCompute && key < p.N;
    // ---- the keeping query blocks: S^T, dP^T, then dV += P^T dO, dK += dS^T Q
    if (issuer) {
      auto load_q = [&](int t) {
        const int st = t & 1, a = M.keep[t];
        mbar_expect_tx(&M.full[st], 2 * TILE);
        for (int ka = 0; ka < 2; ++ka) {
          tma_load_4d(smem + L::ring_off + (2 * st) * TILE + ka * (BM * 128), &tmQ, &M.full[st], ka * 64, h,
                      a * BM, b);
          tma_load_4d(smem + L::ring_off + (2 * st + 1) * TILE + ka * (BM * 128), &tmO, &M.full[st], ka * 64,
                      h, a * BM, b);
        }
      };
      auto issue_S = [&](int t) -> bool {
        const int st = t & 1;
        if (!mbar_wait(&M.full[st], ph_full[st] & 1, abort)) return false;
        ++ph_full[st];
        tc_fence_after();
        const uint32_t sQa = smem_u32(smem + L::ring_off + (2 * st) * TILE);
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + kK_S, desc_kmaj(sK, BN, kk), desc_kmaj(sQa, BM, kk), id_dd, kk > 0);
        mma_commit(&M.s_ready);
        return true;
      };
      auto issue_dP = [&](int t) {
        const uint32_t sOa = smem_u32(smem + L::ring_off + (2 * (t & 1) + 1) * TILE);
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + kK_dP, desc_kmaj(sV, BN, kk), desc_kmaj(sOa, BM, kk), id_dd, kk > 0);
        mma_commit(&M.d_ready);
      };
      for (int t = 0; t < min(nkeep, 2); ++t) load_q(t);
      ok = mbar_wait(&M.load, ph_load & 1, abort);
      if (ok && nkeep > 0 && (ok = issue_S(0))) issue_dP(0);
      // per keeper t: dV += P^T dO and dK's lo part (they read the S^T
      // columns), then S^T(t + 1) over those columns (the next keeper's
      // exponentials need only it), then dK's hi part (it reads the dP^T
      // columns), then dP^T(t + 1) over them
      for (int t = 0; ok && t < nkeep; ++t) {
        const int st = t & 1;
        if (!(ok = mbar_wait(&M.p_ready, ph_p & 1, abort))) break;
        ++ph_p;
        tc_fence_after();
        const uint32_t sQa = smem_u32(smem + L::ring_off + (2 * st) * TILE), sOa = sQa + TILE;
        for (int kk = 0; kk < BM / 16; ++kk) {
          mma_ts(tm + kK_dV, tm + kK_S + kk * 8, desc_mnmaj(sOa, BM, kk), id_pv, (t > 0 || kk > 0) ? 1u : 0u);
          mma_ts(tm + kK_dK, tm + kK_S + 64 + kk * 8, desc_mnmaj(sQa, BM, kk), id_pv, (t > 0 || kk > 0) ? 1u : 0u);
        }
        if (t + 1 < nkeep && !(ok = issue_S(t + 1))) break;
        for (int kk = 0; kk < BM / 16; ++kk)
          mma_ts(tm + kK_dK, tm + kK_dP + kk * 8, desc_mnmaj(sQa, BM, kk), id_pv, 1u);
        mma_commit(&M.empty[st]);
        const uint32_t my = ce[st]++;
        if (t + 1 < nkeep) issue_dP(t + 1);
        if (t + 2 < nkeep) {
          if (!(ok = mbar_wait(&M.empty[st], my & 1, abort))) break;
          load_q(t + 2);
        }
      }
      mma_commit(&M.mma);
    }
    ++ph_load;
    if (tid < kCompute) {
      // Every compute warp runs every iteration (the named barrier below has
      // no bound, so no warp may leave the loop early); after an abort the
      // waits return at once and the work is skipped.
      for (int t = 0; t < nkeep; ++t) {
        const int st = t & 1, a = M.keep[t];
        {  // log-sum-exp (log2 units) and D of the keeper's rows; padding rows get P = 0
          const int nq = a * BM + tid;
          const bool qv = nq < p.N;
          M.lse2[st][tid] = qv ? p.lse[bh * p.N + nq] * 1.4426950408889634f : INFINITY;
          M.Dr[st][tid] = qv ? p.Drow[bh * p.N + nq] : 0.f;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok) ok = wwait(&M.s_ready, ph_s & 1, abort);
        ++ph_s;
        if (!ok) continue;
        tc_fence_after();
        // phase 1 (while dK's hi part and dP^T run): P^T in fp32 over S^T
#pragma unroll 1
        for (int c = 0; c < BM / 32; ++c) {
          uint32_t sv[32];
          tmem_ld32(trow + kK_S + c * 32, sv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            sv[e] = __float_as_uint(fast_exp2(__uint_as_float(sv[e]) * p.scale_log2 - M.lse2[st][c * 32 + e]));
          tmem_st32(trow + kK_S + c * 32, sv);
        }
        tmem_wait_st();
        if (ok) ok = wwait(&M.d_ready, ph_d & 1, abort);
        ++ph_d;
        if (!ok) continue;
        tc_fence_after();
        // phase 2: P^T (bf16) over the read P^T columns [0, 64), dS^T hi over
        // the read dP^T columns [0, 64), dS^T lo (held until every P^T column
        // is read) over columns [64, 128)
        uint32_t dl[64];
#pragma unroll
        for (int c = 0; c < BM / 32; ++c) {
          uint32_t sv[32], dv[32], pp[16], ds[16];
          tmem_ld32(trow + kK_S + c * 32, sv);
          tmem_ld32(trow + kK_dP + c * 32, dv);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int q0 = c * 32 + 2 * e;
            const float p0 = __uint_as_float(sv[2 * e]), p1 = __uint_as_float(sv[2 * e + 1]);
            pp[e] = pack_bf16(p0, p1);
            const float d0 = p0 * (__uint_as_float(dv[2 * e]) - M.Dr[st][q0]) * p.scale;
            const float d1 = p1 * (__uint_as_float(dv[2 * e + 1]) - M.Dr[st][q0 + 1]) * p.scale;
            ds[e] = pack_bf16(d0, d1);
            dl[c * 16 + e] = pack_bf16(d0 - bf16_lo(ds[e]), d1 - bf16_hi(ds[e]));
          }
          tmem_st16(trow + kK_S + c * 16, pp);
          tmem_st16(trow + kK_dP + c * 16, ds);
          // S^T columns [64, 96) are read once chunk 2 is, [96, 128) with chunk 3
          if (c == 2) tmem_st32_at<0>(trow + kK_S + 64, dl);
          if (c == 3) tmem_st32_at<32>(trow + kK_S + 96, dl);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&M.p_ready);
      }
      if (ok) ok = wwait(&M.mma, ph_mma & 1, abort);
    }
    ++ph_mma;
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    // ---- key side of the linear branch: dS_b = total - the keepers' dS_U
    int kpt = 0, kpy = 0, kpx = 0;
    float uk[R], psik[R];
    if (tid < kCompute) {
      if (kvalid) coords(key, p.Hg, p.W, kpt, kpy, kpx);
      float sb[R];
#pragma unroll
      for (int r = 0; r < R; ++r) sb[r] = p.dSU_tot[bh * R * D + r * D + tid];
      float zb = tid < R ? p.dzU_tot[bh * R + tid] : 0.f;
      // four keepers' loads in flight per round trip; the subtractions keep
      // the keepers' order
      int t = 0;
      for (; t + 4 <= nkeep; t += 4) {
        float v4[4][R];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float* src = p.dSU + (bh * p.nb + M.keep[t + i]) * R * D;
#pragma unroll
          for (int r = 0; r < R; ++r) v4[i][r] = __ldcg(src + r * D + tid);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int r = 0; r < R; ++r) sb[r] -= v4[i][r];
        if (tid < R)
          for (int i = 0; i < 4; ++i) zb -= p.dzU[(bh * p.nb + M.keep[t + i]) * R + tid];
      }
      for (; t < nkeep; ++t) {
        const size_t st = bh * p.nb + M.keep[t];
#pragma unroll
        for (int r = 0; r < R; ++r) sb[r] -= p.dSU[st * R * D + r * D + tid];
        if (tid < R) zb -= p.dzU[st * R + tid];
      }
      if (tid < R) M.zb[tid] = zb;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        uint16_t hi, lo;
        split_bf16(sb[r], hi, lo);
        *reinterpret_cast<uint16_t*>(smem + L::sb_off + sw128_off(r, tid, R)) = hi;
        *reinterpret_cast<uint16_t*>(smem + L::sb_off + R * D * 2 + sw128_off(r, tid, R)) = lo;
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (issuer) {
      if (ok) {
        tc_fence_after();
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + kK_S, desc_kmaj(sK, BN, kk), desc_kmaj(sPT, R, kk), id_qr, kk > 0);
      }
      mma_commit(&M.mma);
    }
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort) && ok;
      tc_fence_after();
      uint32_t v[32];
      if (R == 32) tmem_ld32(trow + kK_S, v);
      else tmem_ld16(trow + kK_S, *reinterpret_cast<uint32_t(*)[16]>(v));
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < R; ++i) {
        uk[i] = kvalid ? __uint_as_float(v[i]) : 0.f;
        psik[i] = phi_fast(uk[i]);
      }
#pragma unroll
      for (int pr = 0; pr < R / 2; ++pr) {
        float cs, sn;
        rope_cs(p, M.tab, pr, kpt, kpy, kpx, cs, sn);
        const float r0 = kvalid ? psik[2 * pr] * cs - psik[2 * pr + 1] * sn : 0.f;
        const float r1 = kvalid ? psik[2 * pr] * sn + psik[2 * pr + 1] * cs : 0.f;
        uint16_t h0, l0, h1, l1;
        split_bf16(r0, h0, l0);
        split_bf16(r1, h1, l1);
        const uint32_t off = core_off<R>(tid, 2 * pr);
        *reinterpret_cast<uint32_t*>(smem + L::rho_off + off) = h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t*>(smem + L::rho_off + BN * R * 2 + off) = l0 | ((uint32_t)l1 << 16);
      }
    }
    ++ph_mma;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // dV += rho_k dS_b;  drho_k = V dS_b^T
    if (issuer) {
      if (ok) {
        tc_fence_after();
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint64_t ah = desc_core<R>(sRho, kk), al = desc_core<R>(sRho + BN * R * 2, kk);
          const uint64_t bh_ = desc_mnmaj(sSb, R, kk), bl_ = desc_mnmaj(sSb + R * D * 2, R, kk);
          const uint32_t acc0 = (nkeep > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tm + kK_dV, ah, bh_, id_pv, acc0);
          mma_ss(tm + kK_dV, ah, bl_, id_pv, 1);
          mma_ss(tm + kK_dV, al, bh_, id_pv, 1);
        }
        for (int kk = 0; kk < D / 16; ++kk) {
          mma_ss(tm + kK_S + 32, desc_kmaj(sV, BN, kk), desc_kmaj(sSb, R, kk), id_qr, kk > 0);
          mma_ss(tm + kK_S + 32, desc_kmaj(sV, BN, kk), desc_kmaj(sSb + R * D * 2, R, kk), id_qr, 1);
        }
      }
      mma_commit(&M.mma);
    }
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort) && ok;
      tc_fence_after();
      uint32_t w[32];
      if (R == 32) tmem_ld32(trow + kK_S + 32, w);
      else tmem_ld16(trow + kK_S + 32, *reinterpret_cast<uint32_t(*)[16]>(w));
      tmem_wait_ld();
#pragma unroll
      for (int pr = 0; pr < R / 2; ++pr) {
        float cs, sn;
        rope_cs(p, M.tab, pr, kpt, kpy, kpx, cs, sn);
        const float d0 = __uint_as_float(w[2 * pr]), d1 = __uint_as_float(w[2 * pr + 1]);
        const float p0 = M.zb[2 * pr] + d0 * cs + d1 * sn;
        const float p1 = M.zb[2 * pr + 1] - d0 * sn + d1 * cs;
        const float du0 = kvalid ? p0 * (uk[2 * pr] > 0.f ? 1.f : psik[2 * pr]) : 0.f;
        const float du1 = kvalid ? p1 * (uk[2 * pr + 1] > 0.f ? 1.f : psik[2 * pr + 1]) : 0.f;
        uint16_t h0, l0, h1, l1;
        split_bf16(du0, h0, l0);
        split_bf16(du1, h1, l1);
        const uint32_t off = core_off<R>(tid, 2 * pr);
        *reinterpret_cast<uint32_t*>(smem + L::du_off + off) = h0 | ((uint32_t)h1 << 16);
        *reinterpret_cast<uint32_t*>(smem + L::du_off + BN * R * 2 + off) = l0 | ((uint32_t)l1 << 16);
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + sw128_off(2 * pr, tid, R)) = h0;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + sw128_off(2 * pr + 1, tid, R)) = h1;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + R * BN * 2 + sw128_off(2 * pr, tid, R)) = l0;
        *reinterpret_cast<uint16_t*>(smem + L::dut_off + R * BN * 2 + sw128_off(2 * pr + 1, tid, R)) = l1;
      }
    }
    ++ph_mma;
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    // dK += du P_h^T;  P_h partial = K^T du
    if (issuer) {
      if (ok) {
        tc_fence_after();
        for (int kk = 0; kk < R / 16; ++kk) {
          const uint32_t acc0 = (nkeep > 0 || kk > 0) ? 1u : 0u;
          mma_ss(tm + kK_dK, desc_core<R>(sDu, kk), desc_core<R>(sPC, kk), id_dd, acc0);
          mma_ss(tm + kK_dK, desc_core<R>(sDu + BN * R * 2, kk), desc_core<R>(sPC, kk), id_dd, 1);
        }
        for (int kk = 0; kk < BN / 16; ++kk) {
          mma_ss(tm + kK_dP, desc_mnmaj(sK, BN, kk), desc_kmaj(sDut, R, kk), id_tr, kk > 0);
          mma_ss(tm + kK_dP, desc_mnmaj(sK, BN, kk), desc_kmaj(sDut + R * BN * 2, R, kk), id_tr, 1);
        }
      }
      mma_commit(&M.mma);
    }
    if (tid < kCompute) {
      ok = wwait(&M.mma, ph_mma & 1, abort) && ok;
      tc_fence_after();
      uint32_t t32[32];
      if (R == 32) tmem_ld32(trow + kK_dP, t32);
      else tmem_ld16(trow + kK_dP, *reinterpret_cast<uint32_t(*)[16]>(t32));
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < R; ++i) dph[i] += __uint_as_float(t32[i]);
      // dv, dk rows of the valid keys
      uint16_t* dvr = p.dv + ((b * (size_t)p.N + (kvalid ? key : 0)) * p.H + h) * D;
      uint16_t* dkr = p.dk + ((b * (size_t)p.N + (kvalid ? key : 0)) * p.H + h) * D;
#pragma unroll 1
      for (int c = 0; c < 2 * (D / 32); ++c) {
        const bool isk = c >= D / 32;
        const int cc = isk ? c - D / 32 : c;
        uint32_t v[32];
        tmem_ld32(trow + (isk ? kK_dK : kK_dV) + cc * 32, v);
        tmem_wait_ld();
        if (kvalid && ok) {
          uint4* d4 = reinterpret_cast<uint4*>((isk ? dkr : dvr) + cc * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            d4[q4] = make_uint4(pack_bf16(__uint_as_float(v[8 * q4]), __uint_as_float(v[8 * q4 + 1])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 2]), __uint_as_float(v[8 * q4 + 3])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 4]), __uint_as_float(v[8 * q4 + 5])),
                                pack_bf16(__uint_as_float(v[8 * q4 + 6]), __uint_as_float(v[8 * q4 + 7])));
        }
      }
    }
    ++ph_mma;
    tc_fence_before();
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
  }
  if (tid < kCompute) {
    float* dst = p.dP_part + ((bh * (p.chunks_q + p.chunks_k)) + p.chunks_q + chunk) * D * R + tid * R;
#pragma unroll
    for (int i = 0; i < R; ++i) dst[i] = dph[i];
  }
  if (issuer) {
    mma_commit(&M.mma);
    int no_abort = 0;
    mbar_wait(&M.mma, ph_mma & 1, &no_abort);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  if (tid == 0 && p.dev_err && M.abort) atomicOr(p.dev_err, ROLA_DEVERR_TIMEOUT);
}

// ================================================================ reductions
// dP_h[h] = sum over batches and CTAs of the partials, dgate[h] = sum of the
// gate partials, both in a fixed order (float64).
__global__ void bwd_reduce_kernel(const float* __restrict__ dP_part, const float* __restrict__ dg_part, int B,
                                  int H, int parts, int gparts, int dr, float* __restrict__ dP,
                                  float* __restrict__ dgate) {
  const int h = blockIdx.x;
  for (int e = threadIdx.x; e < dr; e += blockDim.x) {
    double acc = 0.0;
    for (int b = 0; b < B; ++b)
      for (int c = 0; c < parts; ++c) acc += dP_part[(((size_t)b * H + h) * parts + c) * dr + e];
    dP[(size_t)h * dr + e] = (float)acc;
  }
  if (threadIdx.x == 0) {
    double acc = 0.0;
    for (int b = 0; b < B; ++b)
      for (int c = 0; c < gparts; ++c) acc += dg_part[((size_t)b * H + h) * gparts + c];
    dgate[h] = (float)acc;
  }
}

constexpr int kChunk = 8;  // query (or key) blocks per CTA

// Workspace of the backward: transposed mask, per-query-block dS_U and dz_U,
// their totals, D per row, and the partials of dP_h and dgate.
struct BwdWs {
  size_t mt_off, mt_rows, dSU, dzU, dSU_tot, dzU_tot, Drow, dP_part, dg_part, total;
  int cq, ck;
};
static BwdWs bwd_ws(const rola_shape_t* s) {
  using rola_internal::round_up;
  BwdWs w{};
  const size_t nb = (size_t)rola_num_blocks(s), BH = (size_t)s->B * s->H;
  w.cq = w.ck = (int)((nb + kChunk - 1) / kChunk);
  size_t off = 0;
  w.mt_off = off; off += round_up(BH * (nb + 1) * 4, 256);
  w.mt_rows = off; off += round_up(BH * nb * s->k_b * 4, 256);
  w.dSU = off; off += round_up(BH * nb * s->r * s->d * 4, 256);
  w.dzU = off; off += round_up(BH * nb * s->r * 4, 256);
  w.dSU_tot = off; off += round_up(BH * s->r * s->d * 4, 256);
  w.dzU_tot = off; off += round_up(BH * s->r * 4, 256);
  w.Drow = off; off += round_up(BH * (size_t)s->N * 4, 256);
  w.dP_part = off; off += round_up(BH * (size_t)(w.cq + w.ck) * s->d * s->r * 4, 256);
  w.dg_part = off; off += round_up(BH * (size_t)w.cq * 4, 256);
  w.total = off;
  return w;
}

static bool bwd_supports(const rola_shape_t* s) {
  return s->d == D && s->block == BN && (s->r == 16 || s->r == 32) && s->k_b <= kMaxKept &&
         rola_num_blocks(s) <= kMaxBlocks;
}

template <int R>
static rola_status_t launch_bwd(const rola_shape_t* s, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const uint16_t* dout, Params prm, const BwdWs& W, char* base, cudaStream_t cs) {
  CUtensorMap mq, mk, mv, mo;
  if (!rola_host::make_act_map(&mq, q, s, 128) || !rola_host::make_act_map(&mk, k, s, 128) ||
      !rola_host::make_act_map(&mv, v, s, 128) || !rola_host::make_act_map(&mo, dout, s, 128))
    return ROLA_ERR_CUDA;
  const int nb = prm.nb;
  const size_t mt_smem = (size_t)nb * ((nb + 31) / 32) * 4 + (size_t)(nb + 1) * 4;
  if (cudaFuncSetAttribute(mask_t_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)mt_smem) != cudaSuccess)
    return ROLA_ERR_CUDA;
  mask_t_kernel<<<s->B * s->H, 512, mt_smem, cs>>>(prm.idx, nb, prm.kb, reinterpret_cast<int32_t*>(base + W.mt_off),
                                                  reinterpret_cast<int32_t*>(base + W.mt_rows), prm.dev_err);
  const size_t qsmem = QLayout<R>::misc_off + sizeof(QMisc) + 1024;
  const size_t ksmem = KLayout<R>::misc_off + sizeof(KMisc) + 1024;
  if (cudaFuncSetAttribute(bwd_query_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)qsmem) !=
          cudaSuccess ||
      cudaFuncSetAttribute(bwd_key_kernel<R>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ksmem) !=
          cudaSuccess)
    return ROLA_ERR_CUDA;
  bwd_query_kernel<R><<<dim3(W.cq, s->H, s->B), kThreads, qsmem, cs>>>(mq, mk, mv, mo, prm);
  if (cudaGetLastError() != cudaSuccess) return ROLA_ERR_CUDA;
  rola_status_t st = launch_states_total(s, prm.dSU, prm.dzU, const_cast<float*>(prm.dSU_tot),
                                         const_cast<float*>(prm.dzU_tot), cs);
  if (st != ROLA_OK) return st;
  bwd_key_kernel<R><<<dim3(W.ck, s->H, s->B), kThreads, ksmem, cs>>>(mq, mk, mv, mo, prm);
  if (cudaGetLastError() != cudaSuccess) return ROLA_ERR_CUDA;
  return ROLA_OK;
}

}  // namespace bwd
}  // namespace rola

using namespace rola;

extern "C" size_t rola_attention_bwd_workspace_bytes(const rola_shape_t* s) {
  if (rola_internal::check_shape(s) != ROLA_OK || !bwd::bwd_supports(s)) return 0;
  return bwd::bwd_ws(s).total;
}

extern "C" rola_status_t rola_attention_bwd(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                            const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                            const float* S_blk, const float* z_blk, const float* S_glb,
                                            const float* z_glb, const float* gate, const uint16_t* out,
                                            const uint16_t* out_lo, const float* lse, const float* den,
                                            const uint16_t* dout,
                                            uint16_t* dq, uint16_t* dk, uint16_t* dv, float* dP, float* dgate,
                                            void* ws, size_t ws_bytes, int32_t* dev_err, void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q || !k || !v || !idx || !P || !S_blk || !z_blk || !S_glb || !z_glb || !gate || !out || !out_lo || !lse ||
      !den || !dout || !dq || !dk || !dv || !dP || !dgate)
    return ROLA_ERR_INVALID_ARG;
  if (!bwd::bwd_supports(s)) return ROLA_ERR_UNSUPPORTED;
  const void* a16[] = {q, k, v, out, out_lo, dout, dq, dk, dv};
  for (const void* ptr : a16)
    if (!rola_host::aligned(ptr, 16)) return ROLA_ERR_ALIGNMENT;
  const void* a4[] = {idx, S_blk, z_blk, S_glb, z_glb, gate, lse, den, dP, dgate};
  for (const void* ptr : a4)
    if (!rola_host::aligned(ptr, 4)) return ROLA_ERR_ALIGNMENT;
  const bwd::BwdWs W = bwd::bwd_ws(s);
  if (!ws || ws_bytes < W.total || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  char* base = reinterpret_cast<char*>(ws);
  bwd::Params prm{};
  prm.B = s->B;
  prm.H = s->H;
  prm.N = s->N;
  prm.nb = rola_num_blocks(s);
  prm.kb = s->k_b;
  prm.T = s->T;
  prm.Hg = s->Hg;
  prm.W = s->W;
  prm.scale = (float)(1.0 / sqrt((double)s->d));
  prm.scale_log2 = (float)(1.4426950408889634 / sqrt((double)s->d));
  prm.chunk = bwd::kChunk;
  prm.P = P;
  prm.gate = gate;
  prm.idx = idx;
  prm.S_blk = S_blk;
  prm.z_blk = z_blk;
  prm.S_glb = S_glb;
  prm.z_glb = z_glb;
  prm.out = out;
  prm.out_lo = out_lo;
  prm.dout = dout;
  prm.lse = lse;
  prm.den = den;
  prm.mt_off = reinterpret_cast<int32_t*>(base + W.mt_off);
  prm.mt_rows = reinterpret_cast<int32_t*>(base + W.mt_rows);
  prm.dSU = reinterpret_cast<float*>(base + W.dSU);
  prm.dzU = reinterpret_cast<float*>(base + W.dzU);
  prm.dSU_tot = reinterpret_cast<float*>(base + W.dSU_tot);
  prm.dzU_tot = reinterpret_cast<float*>(base + W.dzU_tot);
  prm.Drow = reinterpret_cast<float*>(base + W.Drow);
  prm.dq = dq;
  prm.dk = dk;
  prm.dv = dv;
  prm.dP_part = reinterpret_cast<float*>(base + W.dP_part);
  prm.dg_part = reinterpret_cast<float*>(base + W.dg_part);
  prm.chunks_q = W.cq;
  prm.chunks_k = W.ck;
  prm.dev_err = dev_err;
  rola_host::rope_frequencies(s->r, s->rope_base, prm.rope.freq, prm.rope.axis);
  rola_host::RopeTabLayout tl;
  rola_host::rope_table_layout(s, prm.rope.axis, &tl);
  if (tl.entries > bwd::kTabCap) return ROLA_ERR_UNSUPPORTED;
  for (int i = 0; i < 16; ++i) {
    prm.tab_base[i] = tl.base[i];
    prm.tab_stride[i] = tl.stride[i];
  }
  for (int i = 0; i < 17; ++i) prm.tab_first[i] = tl.first[i];
  prm.tab_entries = tl.entries;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  st = s->r == 32 ? bwd::launch_bwd<32>(s, q, k, v, dout, prm, W, base, cs)
                  : bwd::launch_bwd<16>(s, q, k, v, dout, prm, W, base, cs);
  if (st != ROLA_OK) return st;
  bwd::bwd_reduce_kernel<<<s->H, 256, 0, cs>>>(prm.dP_part, prm.dg_part, s->B, s->H, W.cq + W.ck, W.cq,
                                              s->d * s->r, dP, dgate);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}
