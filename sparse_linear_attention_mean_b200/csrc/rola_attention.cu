// RoLA attention forward on sm_100a: block-sparse softmax branch on the
// 5th-generation tensor cores plus the rotary low-rank linear branch fused
// into the epilogue.
//
// SparkDiffusion write-up (0539edu.com news page), section 05: the sparse
// branch keeps the high-energy query-key blocks and the rotary low-rank linear
// branch restores what sparsification dropped; section 01: at 97 % sparsity
// only 3 % of the blocks are computed, so the kernel has to turn those few
// blocks into dense tensor-core work.
//
// One CTA = one 128-row query tile of one (batch, head): one query block of
// 128 tokens, or two of 64 (then the CTA walks the union of both kept lists
// and masks per row half).  Roles (12 warps):
//   warp 8      TMA producer: Q once, then K_j / V_j of each kept block,
//               gathered by block index into a 2-stage ring (128B swizzle)
//   warp 9      MMA issuer (one thread): S_j = Q K_j^T into tensor memory
//               (two S buffers), O += P_j V_j with P_j read from tensor
//               memory, the q P_h projection and the linear numerator
//   warps 4-7   softmax: thread i owns query row i; online max / sum, bf16 P
//               written back over its S buffer
//   warps 0-3   correction: rescales O in tensor memory when the row max
//               moves, builds the query features rho_q, and writes the output
//   warps 10-11 state gather: S_U = S - sum_{kept} S_j, z_U likewise
// Every wait is bounded; a timeout sets ROLA_DEVERR_TIMEOUT and the CTA
// drains its copies and MMAs, frees tensor memory and returns.
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {

constexpr int kAttnThreads = 384;
constexpr int kMaxKept = 1024;  // k_b limit per query block

template <int D, int BN, int R>
struct AttnLayout {
  static constexpr int BM = 128;
  static constexpr int QB = BM / BN;  // query blocks per tile
  static constexpr int NS = 2;        // K/V ring depth
  static constexpr int KA = D / 64;   // 128-byte swizzle atoms along d
  static constexpr uint32_t Q_BYTES = BM * D * 2;
  static constexpr uint32_t KV_BYTES = BN * D * 2;
  static constexpr uint32_t PT_BYTES = 32 * D * 2;
  static constexpr uint32_t RHO_BYTES = BM * R * 2;
  static constexpr uint32_t SU_BYTES = D * R * 2;
  static constexpr uint32_t CORE_SBO = (R / 8) * 128;  // no-swizzle K-major: 8-row group stride
  static constexpr uint32_t q_off = 0;
  static constexpr uint32_t k_off = q_off + Q_BYTES;
  static constexpr uint32_t v_off = k_off + NS * KV_BYTES;
  static constexpr uint32_t pt_off = v_off + NS * KV_BYTES;
  static constexpr uint32_t rho_off = pt_off + PT_BYTES;   // hi then lo
  static constexpr uint32_t su_off = rho_off + 2 * RHO_BYTES;  // [QB][hi, lo]
  static constexpr uint32_t misc_off = (su_off + QB * 2 * SU_BYTES + 1023) / 1024 * 1024;
  // tensor memory columns
  static constexpr uint32_t S_COL0 = 0;
  static constexpr uint32_t P_OFF = BN / 2;  // bf16 P overwrites the upper half of its S buffer
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t QT_COL = 2 * BN + D;
  static constexpr uint32_t L_COL = 0;  // linear numerator (QB x D columns) after the loop
  static constexpr uint32_t TMEM_COLS = (QT_COL + 32 <= 256) ? 256 : 512;
  static_assert(QB * D <= 2 * BN, "linear numerator must fit in the S buffers");
  static_assert(pt_off % 1024 == 0, "swizzled tiles need 1024-byte alignment");
};

template <int QB>
struct AttnMisc {
  uint64_t bar_q, qt_full, lin_ready, l_done, stats_ready, mma_final, o_ready, pv_done;
  uint64_t k_full[2], v_full[2], kv_empty[2], s_full[2], p_full[2], scale_ready[2];
  uint32_t tmem_base;
  int abort;
  int err;
  int nk;
  int cnt[QB];
  int lin_empty[QB];
  float scale[2][128];
  float rowl[128];
  float zU[QB][32];
  int raw[QB][kMaxKept];
  int ulist[QB * kMaxKept];
  uint8_t umask[QB * kMaxKept];
};

struct AttnParams {
  int N, H, nb, kb, Hg, W;
  float scale_log2;
  const int32_t* idx;
  const uint16_t* P;
  const float* S_blk;
  const float* z_blk;
  const float* S_glb;
  const float* z_glb;
  const float* gate;
  uint16_t* out;
  int32_t* dev_err;
  uint64_t wait_ns;  // bound of each pipeline wait (0: give up at the first wait that finds its stage not ready)
  const int32_t* kb_h;  // per-head kept counts (NULL: kb for every head); idx rows keep stride kb
  RopeTable rope;
};

// All lanes wait; the warp agrees on the outcome (and reconverges).
ROLA_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}

// K-major operand with 128-byte swizzle: `rows` rows of 128-byte atoms, d in
// atoms of 64 elements; k-step kk covers elements [16kk, 16kk + 16).
ROLA_DEV uint64_t desc_kmajor_sw128(uint32_t base, int rows, int kk) {
  return smem_desc(base + (uint32_t)(kk >> 2) * rows * 128 + (uint32_t)(kk & 3) * 32, 16, 1024,
                   kSwizzle128B);
}

template <int D, int BN, int R>
__global__ void __launch_bounds__(kAttnThreads, 1)
    rola_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnLayout<D, BN, R>;
  constexpr int QB = L::QB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  AttnMisc<QB>& M = *reinterpret_cast<AttnMisc<QB>*>(smem + L::misc_off);

  const int tile = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t bh = (size_t)b * p.H + h;

  // A CTA that already timed out in this launch makes the rest skip their
  // work; the barrier gives every thread of the CTA the same answer.
  if (__syncthreads_or(tid == 0 && p.dev_err &&
                       (*reinterpret_cast<volatile int32_t*>(p.dev_err) & ROLA_DEVERR_TIMEOUT)))
    return;
  const uint64_t lim = p.wait_ns;  // bound of each pipeline wait

  // ------------------------------------------------------------ set-up
  if (tid == 0) {
    mbar_init(&M.bar_q, 1);
    mbar_init(&M.qt_full, 1);
    mbar_init(&M.lin_ready, 128 + 64);
    mbar_init(&M.l_done, 1);
    mbar_init(&M.stats_ready, 128);
    mbar_init(&M.mma_final, 1);
    mbar_init(&M.o_ready, 128);
    mbar_init(&M.pv_done, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&M.k_full[i], 1);
      mbar_init(&M.v_full[i], 1);
      mbar_init(&M.kv_empty[i], 1);
      mbar_init(&M.s_full[i], 1);
      mbar_init(&M.p_full[i], 128);
      mbar_init(&M.scale_ready[i], 128);
    }
    M.abort = 0;
    M.err = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&M.tmem_base, L::TMEM_COLS);
    tmem_relinquish();
  }
  // this head's kept count (a count outside [1, kb] is clamped and reported)
  const int kb_want = p.kb_h ? p.kb_h[h] : p.kb;
  const int kbh = min(max(kb_want, 1), p.kb);
  for (int i = tid; i < QB * kbh; i += kAttnThreads) {
    const int qb = i / kbh, a = tile * QB + qb;
    M.raw[qb][i % kbh] = a < p.nb ? p.idx[(bh * p.nb + a) * p.kb + i % kbh] : -1;
  }
  // P_h^T as a K-major (N = r rows, K = d) operand with 128-byte swizzle.
  {
    uint8_t* pt = smem + L::pt_off;
    for (int e = tid; e < R * D; e += kAttnThreads) {
      const int c = e / R, rr = e % R;
      const uint16_t val = p.P[((size_t)h * D + c) * R + rr];
      const int byte = (c & 63) * 2;
      const int chunk = (byte >> 4) ^ (rr & 7);
      *reinterpret_cast<uint16_t*>(pt + (c >> 6) * (32 * 128) + rr * 128 + chunk * 16 + (byte & 15)) =
          val;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    // Validate each kept list (in range, strictly ascending; bad entries are
    // skipped and reported) and merge them into one ascending union.
    int pos[QB], prev[QB], len[QB];
    for (int qb = 0; qb < QB; ++qb) {
      pos[qb] = 0;
      prev[qb] = -1;
      M.cnt[qb] = 0;
      len[qb] = (tile * QB + qb) < p.nb ? kbh : 0;
    }
    int nk = 0, err = kbh != kb_want;
    while (true) {
      int best = 0x7fffffff;
      for (int qb = 0; qb < QB; ++qb) {
        while (pos[qb] < len[qb]) {
          const int v = M.raw[qb][pos[qb]];
          if (v < 0 || v >= p.nb || v <= prev[qb]) {
            err = 1;
            ++pos[qb];
            continue;
          }
          break;
        }
        if (pos[qb] < len[qb]) best = min(best, M.raw[qb][pos[qb]]);
      }
      if (best == 0x7fffffff) break;
      uint8_t mask = 0;
      for (int qb = 0; qb < QB; ++qb)
        if (pos[qb] < len[qb] && M.raw[qb][pos[qb]] == best) {
          mask |= (uint8_t)(1u << qb);
          prev[qb] = best;
          ++pos[qb];
          ++M.cnt[qb];
        }
      M.ulist[nk] = best;
      M.umask[nk] = mask;
      ++nk;
    }
    for (int qb = 0; qb < QB; ++qb) M.lin_empty[qb] = M.cnt[qb] >= p.nb;
    M.nk = nk;
    M.err = err;
  }
  __syncthreads();
  const uint32_t tm = M.tmem_base;
  const int nk = M.nk;
  volatile int* abort = &M.abort;

  if (warp == 8) {
    // -------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_expect_tx(&M.bar_q, L::Q_BYTES);
      for (int ka = 0; ka < L::KA; ++ka)
        tma_load_4d(smem + L::q_off + ka * (L::BM * 128), &tmQ, &M.bar_q, ka * 64, h, tile * L::BM, b);
      int j = 0;
      for (; j < nk; ++j) {
        const int st = j % L::NS;
        if (j >= L::NS && !mbar_wait(&M.kv_empty[st], ((j / L::NS) - 1) & 1, abort, lim)) break;
        const int u = M.ulist[j];
        mbar_expect_tx(&M.k_full[st], L::KV_BYTES);
        for (int ka = 0; ka < L::KA; ++ka)
          tma_load_4d(smem + L::k_off + st * L::KV_BYTES + ka * (BN * 128), &tmK, &M.k_full[st],
                      ka * 64, h, u * BN, b);
        mbar_expect_tx(&M.v_full[st], L::KV_BYTES);
        for (int ka = 0; ka < L::KA; ++ka)
          tma_load_4d(smem + L::v_off + st * L::KV_BYTES + ka * (BN * 128), &tmV, &M.v_full[st],
                      ka * 64, h, u * BN, b);
      }
      // Drain: copies complete on their own; wait (bounded) for the last ones.
      int no_abort = 0;
      mbar_wait(&M.bar_q, 0, &no_abort);
      for (int i = (j > L::NS ? j - L::NS : 0); i < j; ++i) {
        mbar_wait(&M.k_full[i % L::NS], (i / L::NS) & 1, &no_abort);
        mbar_wait(&M.v_full[i % L::NS], (i / L::NS) & 1, &no_abort);
      }
      if (no_abort) *abort = 1;
    }
  } else if (warp == 9) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, BN);
      constexpr uint32_t idesc_pv = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, D);
      constexpr uint32_t idesc_qt = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, R);
      constexpr uint32_t idesc_l = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, D);
      const uint32_t sQ = smem_u32(smem + L::q_off);
      const uint32_t sK = smem_u32(smem + L::k_off);
      const uint32_t sV = smem_u32(smem + L::v_off);
      const uint32_t sPT = smem_u32(smem + L::pt_off);
      const uint32_t sRho = smem_u32(smem + L::rho_off);
      const uint32_t sSU = smem_u32(smem + L::su_off);

      auto issue_pv = [&](int i) -> bool {
        const int sb = i & 1, st = i % L::NS;
        if (!mbar_wait(&M.p_full[sb], (i >> 1) & 1, abort, lim)) return false;
        if (!mbar_wait(&M.o_ready, i & 1, abort, lim)) return false;
        if (!mbar_wait(&M.v_full[st], (i / L::NS) & 1, abort, lim)) return false;
        tc_fence_after();
        const uint32_t vbase = sV + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = smem_desc(vbase + kk * 16 * 128, BN * 128, 1024, kSwizzle128B);
          mma_ts(tm + L::O_COL, tm + L::S_COL0 + sb * BN + L::P_OFF + kk * 8, bdesc, idesc_pv,
                 (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&M.kv_empty[st]);
        mma_commit(&M.pv_done);
        return true;
      };

      bool ok = mbar_wait(&M.bar_q, 0, abort, lim);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + L::QT_COL, desc_kmajor_sw128(sQ, L::BM, kk), desc_kmajor_sw128(sPT, 32, kk),
                 idesc_qt, kk > 0 ? 1u : 0u);
        mma_commit(&M.qt_full);
      }
      for (int j = 0; ok && j < nk; ++j) {
        const int st = j % L::NS, sb = j & 1;
        ok = mbar_wait(&M.k_full[st], (j / L::NS) & 1, abort, lim);
        // The S buffer about to be overwritten still holds P_{j-2}; let that
        // P.V finish first.
        if (ok && j >= 2) ok = mbar_wait(&M.pv_done, (j - 2) & 1, abort, lim);
        if (!ok) break;
        tc_fence_after();
        const uint32_t kbase = sK + st * L::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tm + L::S_COL0 + sb * BN, desc_kmajor_sw128(sQ, L::BM, kk),
                 desc_kmajor_sw128(kbase, BN, kk), idesc_s, kk > 0 ? 1u : 0u);
        mma_commit(&M.s_full[sb]);
        if (j >= 1) ok = issue_pv(j - 1);
      }
      if (ok && nk > 0) ok = issue_pv(nk - 1);
      if (ok) ok = mbar_wait(&M.lin_ready, 0, abort, lim);
      if (ok && nk > 0) ok = mbar_wait(&M.pv_done, (nk - 1) & 1, abort, lim);
      if (ok) {
        tc_fence_after();
#pragma unroll
        for (int qb = 0; qb < QB; ++qb) {
          const uint32_t suh = sSU + qb * 2 * L::SU_BYTES, sul = suh + L::SU_BYTES;
#pragma unroll
          for (int kk = 0; kk < R / 16; ++kk) {
            const uint64_t ah = smem_desc(sRho + kk * 256, 128, L::CORE_SBO, kSwizzleNone);
            const uint64_t al = smem_desc(sRho + L::RHO_BYTES + kk * 256, 128, L::CORE_SBO, kSwizzleNone);
            const uint64_t bh_ = smem_desc(suh + kk * 256, 128, L::CORE_SBO, kSwizzleNone);
            const uint64_t bl_ = smem_desc(sul + kk * 256, 128, L::CORE_SBO, kSwizzleNone);
            const uint32_t dcol = tm + L::L_COL + qb * D;
            mma_ss(dcol, ah, bh_, idesc_l, kk > 0 ? 1u : 0u);
            mma_ss(dcol, ah, bl_, idesc_l, 1u);
            mma_ss(dcol, al, bh_, idesc_l, 1u);
          }
        }
        mma_commit(&M.l_done);
      }
      // Whatever happened, let every issued MMA finish before teardown.
      mma_commit(&M.mma_final);
      int no_abort = 0;
      mbar_wait(&M.mma_final, 0, &no_abort);
      if (no_abort) *abort = 1;
    }
  } else if (warp >= 4 && warp < 8) {
    // -------------------------------------------------------- softmax
    const int row = tid - 128;
    const uint32_t trow = tm + ((uint32_t)((warp & 3) * 32) << 16);
    const int qb = row / BN;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
      const int sb = j & 1;
      if (!warp_wait(&M.s_full[sb], (j >> 1) & 1, abort, lim)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(trow + L::S_COL0 + sb * BN + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_wait_ld();
      const int u = M.ulist[j];
      const bool allowed = (M.umask[j] >> qb) & 1;
      const int valid = allowed ? min(BN, p.N - u * BN) : 0;
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < BN; ++c)
        if (c < valid) mx = fmaxf(mx, __uint_as_float(s[c]));
      const float mnew = fmaxf(m, mx * p.scale_log2);
      const float alpha = (mnew == -INFINITY) ? 1.f : fast_exp2(m - mnew);
      M.scale[sb][row] = alpha;
      mbar_arrive(&M.scale_ready[sb]);
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < BN; c += 2) {
        const float p0 = c < valid ? fast_exp2(fmaf(__uint_as_float(s[c]), p.scale_log2, -mnew)) : 0.f;
        const float p1 =
            c + 1 < valid ? fast_exp2(fmaf(__uint_as_float(s[c + 1]), p.scale_log2, -mnew)) : 0.f;
        sum += p0 + p1;
        s[c >> 1] = pack_bf16(p0, p1);
      }
      l = l * alpha + sum;
      m = mnew;
#pragma unroll
      for (int c = 0; c < BN / 64; ++c)
        tmem_st32(trow + L::S_COL0 + sb * BN + L::P_OFF + c * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&M.p_full[sb]);
    }
    if (ok) {
      M.rowl[row] = l;
      mbar_arrive(&M.stats_ready);
    }
  } else if (warp < 4) {
    // -------------------------------------------------------- correction + epilogue
    const int row = tid;
    const uint32_t trow = tm + ((uint32_t)(warp * 32) << 16);
    const int qb = row / BN;
    const int n = tile * L::BM + row;
    mbar_arrive(&M.o_ready);  // iteration 0: nothing to rescale
    float psi[R];
    bool ok = warp_wait(&M.qt_full, 0, abort, lim);
    if (ok) {
      tc_fence_after();
      uint32_t qt[32];
      if constexpr (R == 32) {
        tmem_ld32(trow + L::QT_COL, qt);
      } else {
        tmem_ld16(trow + L::QT_COL, *reinterpret_cast<uint32_t(*)[16]>(&qt[0]));
      }
      tmem_wait_ld();
      const int nn = n < p.N ? n : p.N - 1;
      const int pt = nn / (p.Hg * p.W), py = (nn / p.W) % p.Hg, px = nn % p.W;
      uint8_t* rho_hi = smem + L::rho_off;
      uint8_t* rho_lo = rho_hi + L::RHO_BYTES;
      const uint32_t rbase = (row >> 3) * L::CORE_SBO + (row & 7) * 16;
#pragma unroll
      for (int pr = 0; pr < R / 2; ++pr) {
        const float x0 = phi(__uint_as_float(qt[2 * pr]));
        const float x1 = phi(__uint_as_float(qt[2 * pr + 1]));
        psi[2 * pr] = x0;
        psi[2 * pr + 1] = x1;
        const int ax = p.rope.axis[pr];
        float sn, cs;
        rope_sincos(ax == 0 ? pt : (ax == 1 ? py : px), p.rope.freq[pr], &sn, &cs);
        const float r0 = x0 * cs - x1 * sn, r1 = x0 * sn + x1 * cs;
        const uint32_t hi = pack_bf16(r0, r1);
        const uint32_t lo = pack_bf16(r0 - bf16_lo(hi), r1 - bf16_hi(hi));
        const int c = 2 * pr;
        const uint32_t off = rbase + (c >> 3) * 128 + (c & 7) * 2;
        *reinterpret_cast<uint32_t*>(rho_hi + off) = hi;
        *reinterpret_cast<uint32_t*>(rho_lo + off) = lo;
      }
      fence_proxy_async_smem();
      mbar_arrive(&M.lin_ready);
    }
    for (int j = 1; ok && j < nk; ++j) {
      const int sb = j & 1;
      ok = warp_wait(&M.scale_ready[sb], (j >> 1) & 1, abort, lim);
      if (!ok) break;
      const float alpha = M.scale[sb][row];
      ok = warp_wait(&M.pv_done, (j - 1) & 1, abort, lim);
      if (!ok) break;
      tc_fence_after();
      if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(trow + L::O_COL + c * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st32(trow + L::O_COL + c * 32, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&M.o_ready);
    }
    if (ok) ok = warp_wait(&M.stats_ready, 0, abort, lim);
    if (ok && nk > 0) ok = warp_wait(&M.pv_done, (nk - 1) & 1, abort, lim);
    if (ok) ok = warp_wait(&M.l_done, 0, abort, lim);
    if (ok) {
      tc_fence_after();
      const float lsum = M.rowl[row];
      const float inv_l = lsum > 0.f ? 1.f / lsum : 0.f;
      float den = 0.f;
#pragma unroll
      for (int c = 0; c < R; ++c) den = fmaf(psi[c], M.zU[qb][c], den);
      const float lin = (M.lin_empty[qb] || nk == 0) ? 0.f : p.gate[h] / den;
      const bool write = n < p.N;
      uint16_t* orow = p.out + (((size_t)b * p.N + (write ? n : 0)) * p.H + h) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32], lv[32];
        tmem_ld32(trow + L::O_COL + c * 32, o);
        tmem_ld32(trow + L::L_COL + qb * D + c * 32, lv);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float o0 = nk > 0 ? __uint_as_float(o[2 * e]) * inv_l : 0.f;
          const float o1 = nk > 0 ? __uint_as_float(o[2 * e + 1]) * inv_l : 0.f;
          const float y0 = o0 + lin * __uint_as_float(lv[2 * e]);
          const float y1 = o1 + lin * __uint_as_float(lv[2 * e + 1]);
          w[e] = pack_bf16(y0, y1);
        }
        if (write) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
    }
  } else {
    // -------------------------------------------------------- state gather
    const int gt = tid - 320;  // 0..63
    constexpr int E = R * D, PER = E / 256;  // float4 per thread
    const float* Sg = p.S_glb + bh * E;
    const float* zg = p.z_glb + bh * R;
    for (int qb = 0; qb < QB; ++qb) {
      float4 acc[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      float zacc = 0.f;
      for (int j = 0; j < nk; ++j) {
        if (!((M.umask[j] >> qb) & 1)) continue;
        const size_t st = (bh * p.nb + M.ulist[j]);
        const float4* src = reinterpret_cast<const float4*>(p.S_blk + st * E);
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          const float4 x = __ldg(src + gt + 64 * i);
          acc[i].x += x.x;
          acc[i].y += x.y;
          acc[i].z += x.z;
          acc[i].w += x.w;
        }
        if (gt < R) zacc += p.z_blk[st * R + gt];
      }
      uint8_t* su_hi = smem + L::su_off + qb * 2 * L::SU_BYTES;
      uint8_t* su_lo = su_hi + L::SU_BYTES;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const float4 g4 = __ldg(reinterpret_cast<const float4*>(Sg) + gt + 64 * i);
        const float v4[4] = {g4.x - acc[i].x, g4.y - acc[i].y, g4.z - acc[i].z, g4.w - acc[i].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int f = (gt + 64 * i) * 4 + t;
          const int c = f / D, e = f % D;  // S_U[c][e] -> operand row e, k c
          const uint32_t hi = f2bf(v4[t]);
          const uint32_t lo = f2bf(v4[t] - __uint_as_float(hi << 16));
          const uint32_t off = (e >> 3) * L::CORE_SBO + (c >> 3) * 128 + (e & 7) * 16 + (c & 7) * 2;
          *reinterpret_cast<uint16_t*>(su_hi + off) = (uint16_t)hi;
          *reinterpret_cast<uint16_t*>(su_lo + off) = (uint16_t)lo;
        }
      }
      if (gt < R) M.zU[qb][gt] = zg[gt] - zacc;
    }
    fence_proxy_async_smem();
    mbar_arrive(&M.lin_ready);
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tm, L::TMEM_COLS);
  }
  if (tid == 0 && p.dev_err && (M.abort || M.err))
    atomicOr(p.dev_err, (M.abort ? ROLA_DEVERR_TIMEOUT : 0) | (M.err ? ROLA_DEVERR_BAD_INDEX : 0));
}

// ------------------------------------------------------------------ host

static bool make_map(CUtensorMap* m, const void* base, const rola_shape_t* s, int box_rows) {
  auto enc = rola_host::encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)s->d, (cuuint64_t)s->H, (cuuint64_t)s->N, (cuuint64_t)s->B};
  const cuuint64_t strides[3] = {(cuuint64_t)s->d * 2, (cuuint64_t)s->H * s->d * 2,
                                 (cuuint64_t)s->N * s->H * s->d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BN, int R>
static rola_status_t launch_attn(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const AttnParams& prm, cudaStream_t cs) {
  using L = AttnLayout<D, BN, R>;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, q, s, 128) || !make_map(&mk, k, s, BN) || !make_map(&mv, v, s, BN))
    return ROLA_ERR_CUDA;
  const size_t smem = L::misc_off + sizeof(AttnMisc<L::QB>) + 1024;
  auto kern = rola_attn_kernel<D, BN, R>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return ROLA_ERR_CUDA;
  const dim3 grid((s->N + 127) / 128, s->H, s->B);
  kern<<<grid, kAttnThreads, smem, cs>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

// The persistent two-tile kernel (rola_attention_pair.cu) serves d = 128 with
// 128-token blocks and k_b <= 256; this one-tile kernel serves the rest.
bool pair_kernel_supports(const rola_shape_t* s);
rola_status_t launch_pair_kernel(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                 const float* S_blk, const float* z_blk, const float* S_glb,
                                 const float* z_glb, const float* gate, uint16_t* out, int32_t* dev_err,
                                 const int32_t* kb_h, uint64_t wait_ns, float* lse, float* den,
                                 uint16_t* out_lo, cudaStream_t cs);

}  // namespace rola

using namespace rola;

rola_status_t rola::attention_launch(const rola_shape_t* s, const int32_t* kb_h, const uint16_t* q,
                                     const uint16_t* k, const uint16_t* v, const int32_t* idx,
                                     const uint16_t* P, const float* S_blk, const float* z_blk,
                                     const float* S_glb, const float* z_glb, const float* gate,
                                     uint16_t* out, int32_t* dev_err, uint64_t wait_limit_ns,
                                     void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q || !k || !v || !idx || !P || !S_blk || !z_blk || !S_glb || !z_glb || !gate || !out)
    return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(q, 16) || !rola_host::aligned(k, 16) || !rola_host::aligned(v, 16) ||
      !rola_host::aligned(out, 16) || !rola_host::aligned(S_blk, 16) ||
      !rola_host::aligned(S_glb, 16) || !rola_host::aligned(idx, 4) || !rola_host::aligned(P, 2))
    return ROLA_ERR_ALIGNMENT;
  if (s->k_b > kMaxKept) return ROLA_ERR_UNSUPPORTED;
  AttnParams prm{};
  prm.N = s->N;
  prm.H = s->H;
  prm.nb = rola_num_blocks(s);
  prm.kb = s->k_b;
  prm.Hg = s->Hg;
  prm.W = s->W;
  prm.scale_log2 = (float)(1.4426950408889634 / sqrt((double)s->d));
  prm.idx = idx;
  prm.P = P;
  prm.S_blk = S_blk;
  prm.z_blk = z_blk;
  prm.S_glb = S_glb;
  prm.z_glb = z_glb;
  prm.gate = gate;
  prm.out = out;
  prm.dev_err = dev_err;
  prm.wait_ns = wait_limit_ns;
  prm.kb_h = kb_h;
  rola_host::rope_frequencies(s->r, s->rope_base, prm.rope.freq, prm.rope.axis);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  // the two-tile kernel reads the states with 32-byte loads and P_h with 16-byte loads
  if (pair_kernel_supports(s) && rola_host::aligned(S_blk, 32) && rola_host::aligned(S_glb, 32) &&
      rola_host::aligned(P, 16))
    return launch_pair_kernel(s, q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate, out, dev_err, kb_h,
                              wait_limit_ns, nullptr, nullptr, nullptr, cs);
  if (s->d == 128 && s->block == 128 && s->r == 32) return launch_attn<128, 128, 32>(s, q, k, v, prm, cs);
  if (s->d == 128 && s->block == 128 && s->r == 16) return launch_attn<128, 128, 16>(s, q, k, v, prm, cs);
  if (s->d == 64 && s->block == 64 && s->r == 16) return launch_attn<64, 64, 16>(s, q, k, v, prm, cs);
  if (s->d == 64 && s->block == 64 && s->r == 32) return launch_attn<64, 64, 32>(s, q, k, v, prm, cs);
  if (s->d == 64 && s->block == 128 && s->r == 16) return launch_attn<64, 128, 16>(s, q, k, v, prm, cs);
  if (s->d == 64 && s->block == 128 && s->r == 32) return launch_attn<64, 128, 32>(s, q, k, v, prm, cs);
  return ROLA_ERR_UNSUPPORTED;
}

extern "C" rola_status_t rola_attention_fwd_bounded(const rola_shape_t* s, const uint16_t* q,
                                                    const uint16_t* k, const uint16_t* v,
                                                    const int32_t* idx, const uint16_t* P,
                                                    const float* S_blk, const float* z_blk,
                                                    const float* S_glb, const float* z_glb,
                                                    const float* gate, uint16_t* out,
                                                    int32_t* dev_err, uint64_t wait_limit_ns,
                                                    void* stream) {
  return attention_launch(s, nullptr, q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate, out, dev_err,
                          wait_limit_ns, stream);
}

extern "C" rola_status_t rola_attention_fwd(const rola_shape_t* s, const uint16_t* q,
                                            const uint16_t* k, const uint16_t* v,
                                            const int32_t* idx, const uint16_t* P,
                                            const float* S_blk, const float* z_blk,
                                            const float* S_glb, const float* z_glb,
                                            const float* gate, uint16_t* out, int32_t* dev_err,
                                            void* stream) {
  return rola_attention_fwd_bounded(s, q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate, out, dev_err,
                                    kWaitLimitNs, stream);
}

extern "C" rola_status_t rola_attention_fwd_train(const rola_shape_t* s, const uint16_t* q,
                                                  const uint16_t* k, const uint16_t* v,
                                                  const int32_t* idx, const uint16_t* P,
                                                  const float* S_blk, const float* z_blk,
                                                  const float* S_glb, const float* z_glb,
                                                  const float* gate, uint16_t* out, uint16_t* out_lo,
                                                  float* lse, float* den, int32_t* dev_err, void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q || !k || !v || !idx || !P || !S_blk || !z_blk || !S_glb || !z_glb || !gate || !out || !out_lo || !lse ||
      !den)
    return ROLA_ERR_INVALID_ARG;
  if (!pair_kernel_supports(s)) return ROLA_ERR_UNSUPPORTED;
  if (!rola_host::aligned(q, 16) || !rola_host::aligned(k, 16) || !rola_host::aligned(v, 16) ||
      !rola_host::aligned(out, 16) || !rola_host::aligned(S_blk, 32) || !rola_host::aligned(S_glb, 32) ||
      !rola_host::aligned(idx, 4) || !rola_host::aligned(P, 16) || !rola_host::aligned(lse, 4) ||
      !rola_host::aligned(den, 4) || !rola_host::aligned(out_lo, 16))
    return ROLA_ERR_ALIGNMENT;
  return launch_pair_kernel(s, q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate, out, dev_err, nullptr,
                            kWaitLimitNs, lse, den, out_lo, reinterpret_cast<cudaStream_t>(stream));
}
