// RoLA attention forward, persistent two-tile kernel for 128-token blocks and
// d = 128 (the Wan attention shapes).
//
// SparkDiffusion write-up (0539edu.com news page), section 05: the sparse
// branch keeps the high-energy query-key blocks, a rotary low-rank linear
// branch restores the dropped context; section 01: at 97 % sparsity only 3 %
// of the blocks remain, so the kernel must turn few, scattered blocks into
// dense tensor-core work.
//
// A CTA is persistent and works on units: two adjacent query blocks
// (2p, 2p+1) of one (batch, head), one per slot.  Their kept lists overlap
// heavily, so the CTA walks the ascending UNION of both lists; each key block
// is loaded once (TMA, gathered by block index) and multiplied by the query
// tile of every slot that keeps it.  Tensor memory holds S0, S1, O0, O1
// (4 x 128 columns); the bf16 probabilities P overwrite the first 64 columns
// of their S buffer and feed P.V straight from tensor memory.
//
// Warp roles (12 warps, three warpgroups):
//   warps 0-3, 4-7  one slot each (184 registers): softmax -- thread i owns
//                   query row i, loads its 128 scores with one tensor-memory
//                   read, and rescales O lazily (only when the row max grows
//                   by more than 2^8, which keeps P <= 256); at the tile end
//                   rho_q = R(t, y, x) phi(q P_h) (rotary angles from a per-CTA
//                   cos/sin table), psi_q . z_U and rho'_q (below), and the
//                   epilogue out = O / l (tile-end code as rolled loops: it
//                   runs once per unit, cold in the instruction cache)
//   warp 8          producer: the unit lists, built one unit ahead by a
//                   bitmap merge of both kept lists (three list buffers),
//                   Q tiles and the K/V ring (TMA)
//   warp 9          MMA issuer: S = Q K^T, O += P V, q P_h, O += rho'_q S_U
//   warps 10-11     P_h^T in shared memory (rewritten when the head
//                   changes); gather of the linear-branch states of every
//                   union block (32-byte loads that skip L1) into fp32
//                   shared-memory accumulators: S_U = S - sum_kept S_j, z_U
// The linear branch is folded into O: at a tile end the softmax warps write
// rho'_q = rho_q g_h l / (psi_q . z_U) (bf16 hi + lo) into tensor memory and
// one more MMA adds rho'_q S_U to O, S_U coming from the gather warps'
// accumulators converted in place; the epilogue is then out = O / l.  The
// next unit's S MMAs do not wait for that epilogue, only its first P.V does.
// Every wait is bounded; on a timeout the CTA drains its copies and MMAs,
// frees tensor memory and reports ROLA_DEVERR_TIMEOUT.
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {
namespace pairk {

constexpr int kThreads = 384;
constexpr int kMaxKept = 256;           // k_b limit of this kernel
constexpr int kMaxUnion = 2 * kMaxKept;
constexpr int NR = 3;                   // K/V ring slots (each one K or one V tile)
constexpr int D = 128, BM = 128, BN = 128;
constexpr uint32_t TILE = BM * D * 2;   // 32 KB: one Q, K or V tile
constexpr float kRescaleThreshold = 8.f;  // log2 units

template <int R>
struct Layout {
  static constexpr uint32_t q_off = 0;                    // 2 tiles
  static constexpr uint32_t ring_off = q_off + 2 * TILE;  // NR tiles
  static constexpr uint32_t pt_off = ring_off + NR * TILE;
  static constexpr uint32_t PT_BYTES = 32 * D * 2;
  static constexpr uint32_t acc_off = pt_off + PT_BYTES;  // fp32 state accumulators [2][r * d]
  static constexpr uint32_t misc_off = (acc_off + 2 * R * D * 4 + 1023) / 1024 * 1024;
  // S_U (bf16 hi, then lo) replaces a slot's accumulator in place
  static constexpr uint32_t SU_BYTES = R * D * 2;
  static_assert(acc_off % 1024 == 0 && (R * D * 4) % 1024 == 0, "S_U operands need 1024-byte alignment");
  // tensor memory columns
  // S_s at columns [128 s, 128 s + 128), O_s at [256 + 128 s, ...): s_col / o_col

  static constexpr uint32_t P_OFF = 0;  // bf16 P over the first 64 columns of its S buffer
};

constexpr int NL = 3;        // unit lists in flight: the producer builds one unit ahead
constexpr int kMaxBlocks = 1024;  // n_blocks limit (the list merge keeps one bit per block)

constexpr uint16_t kNoBlock = 0xffff;

// One unit's work lists.  The union (ascending, with a per-slot mask) drives
// the state gather.  The steps drive the tensor-core pipeline: in step j slot
// s works on key block sblk[s][j] (kNoBlock: slot idle).  A block both slots
// keep is one shared step (its K and V tiles serve both); the blocks only one
// slot keeps are paired across the slots, each step then loading two K/V
// pairs, so that both slots have a tile in almost every step.
struct UnitList {
  int b, h, a[2];
  int active[2];
  int nu;  // union entries
  int ns;  // steps
  int cnt[2];
  int lin_empty[2];
  uint16_t ulist[kMaxUnion];
  uint8_t umask[kMaxUnion];
  uint16_t sblk[2][kMaxKept];
};

constexpr int kTabCap = 1024;  // cos/sin entries of the rotary table in shared memory

struct Misc {
  uint64_t list_full[NL], list_empty[NL];
  uint64_t q_full[2], q_empty[2];
  uint64_t ring_full[NR], ring_empty[NR];
  uint64_t s_full[2], p_full[2];
  uint64_t pt_full, qt_full[2], zu_ready[2], cvt[2], lin_ready[2], l_done[2], o_free[2];
  uint64_t mma_final;
  uint32_t tmem_base;
  int abort;
  int err;
  float zU[2][32];
  float2 tab[kTabCap];  // (cos, sin) of pos * freq per rotation pair and grid position
  int4 rope_pair[16];   // per rotation pair: table base, stride per position, axis
  uint32_t kept_bits[2][kMaxBlocks / 32];  // list merge scratch of the producer
  UnitList L[NL];
};

struct Params {
  int B, H, N, nb, kb, T, Hg, W, npairs, units;
  float scale_log2;
  const int32_t* idx;
  const uint16_t* P;
  const float* S_blk;
  const float* z_blk;
  const float* S_glb;
  const float* z_glb;
  const float* gate;
  uint16_t* out;
  int out_32b;  // out is 32-byte aligned: the epilogue stores 32 bytes at a time
  int32_t* dev_err;
  uint64_t wait_ns;  // bound of each pipeline wait (0: give up at the first wait that finds its stage not ready)
  const int32_t* kb_h;  // per-head kept counts (NULL: kb for every head); idx rows keep stride kb
  float* lse;  // optional [B, H, N]: natural log-sum-exp of the scaled kept scores per row
  float* den;  // optional [B, H, N]: linear denominator psi_q . z_U (NaN when the complement is empty)
  uint16_t* out_lo;  // optional [B, N, H, d]: bf16 of out (in fp32) minus its bf16 rounding
  RopeTable rope;
  // rotary table: entry of pair pr at position pos = tab_base[pr] + pos * tab_stride[pr];
  // pair pr fills entries [tab_first[pr], tab_first[pr + 1]) of the fill order
  int tab_base[16], tab_stride[16], tab_first[17];
  int tab_entries;
};

ROLA_DEV uint32_t s_col(int s) { return (uint32_t)s * 128u; }
ROLA_DEV uint32_t o_col(int s) { return 256u + (uint32_t)s * 128u; }

ROLA_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint64_t limit_ns) {
  const bool ok = mbar_wait(bar, parity, abort, limit_ns);
  return __all_sync(0xffffffffu, ok);
}
ROLA_DEV uint64_t desc_k_sw128(uint32_t base, int rows, int kk) {
  return smem_desc(base + (uint32_t)(kk >> 2) * rows * 128 + (uint32_t)(kk & 3) * 32, 16, 1024,
                   kSwizzle128B);
}
// Descriptor of k-step kk from the descriptor of k-step 0: only the start
// address field (bits 0-13, in 16-byte units) moves, and shared-memory
// addresses stay below 2^18 bytes, so a plain add cannot carry out of it.
ROLA_DEV constexpr uint64_t kstep_k_sw128(int rows, int kk) {
  return (uint64_t)(((kk >> 2) * rows * 128 + (kk & 3) * 32) >> 4);
}
template <uint32_t N>
ROLA_DEV void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <uint32_t N>
ROLA_DEV void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

// 32-byte read-only load (two float4) that does not allocate in L1: the block
// states are read once per unit and would only evict other lines.
ROLA_DEV void ldg_na8(const float* p, float4& a, float4& b) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(a.x), "=f"(a.y), "=f"(a.z), "=f"(a.w), "=f"(b.x), "=f"(b.y), "=f"(b.z), "=f"(b.w)
               : "l"(p));
}

ROLA_DEV void decode_unit(const Params& p, int id, int& b, int& h, int& pair) {
  pair = id % p.npairs;
  h = (id / p.npairs) % p.H;
  b = id / (p.npairs * p.H);
}

// kLoP (the training forward): P enters P.V as bf16 hi + lo, so that the
// output -- which the backward's D = dout . o_sp is formed from -- carries ~16
// mantissa bits instead of the ~8 of bf16 P.
template <int R, bool kLoP>
__global__ void __launch_bounds__(kThreads, 1)
    rola_attn_pair_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const Params p) {
  using Ly = Layout<R>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Misc& M = *reinterpret_cast<Misc*>(smem + Ly::misc_off);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // A CTA that already timed out in this launch makes the rest skip their
  // work; the barrier gives every thread of the CTA the same answer.
  if (__syncthreads_or(tid == 0 && p.dev_err &&
                       (*reinterpret_cast<volatile int32_t*>(p.dev_err) & ROLA_DEVERR_TIMEOUT)))
    return;
  const uint64_t lim = p.wait_ns;  // bound of each pipeline wait

  if (tid == 0) {
    for (int i = 0; i < NL; ++i) {
      mbar_init(&M.list_full[i], 1);
      mbar_init(&M.list_empty[i], 1 + 2 * 128 + 64);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&M.q_full[i], 1);
      mbar_init(&M.q_empty[i], 1);
      mbar_init(&M.s_full[i], 1);
      mbar_init(&M.p_full[i], 128);
      mbar_init(&M.qt_full[i], 1);
      mbar_init(&M.zu_ready[i], 64);
      mbar_init(&M.cvt[i], 64);
      mbar_init(&M.lin_ready[i], 128);
      mbar_init(&M.l_done[i], 1);
      mbar_init(&M.o_free[i], 128);
    }
    for (int i = 0; i < NR; ++i) {
      mbar_init(&M.ring_full[i], 1);
      mbar_init(&M.ring_empty[i], 1);
    }
    mbar_init(&M.pt_full, 64);
    mbar_init(&M.mma_final, 1);
    M.abort = 0;
    M.err = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&M.tmem_base, 512);
    tmem_relinquish();
  }
  // rotary cos/sin table, once per (persistent) CTA
  if (tid < R / 2) M.rope_pair[tid] = make_int4(p.tab_base[tid], p.tab_stride[tid], p.rope.axis[tid], 0);
  for (int e = tid; e < p.tab_entries; e += kThreads) {
    int pr = 0;
    while (pr + 1 < R / 2 && e >= p.tab_first[pr + 1]) ++pr;
    const int pos = e - p.tab_first[pr];
    float sn, cs;
    rope_sincos(pos, p.rope.freq[pr], &sn, &cs);
    M.tab[p.tab_base[pr] + pos * p.tab_stride[pr]] = make_float2(cs, sn);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = M.tmem_base;
  volatile int* abort = &M.abort;
  const int my_units = p.units > (int)blockIdx.x ? (p.units - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (warp < 8) {
    // ================================================================ one slot: softmax, rho_q, epilogue
    setmaxnreg_inc<184>();
    const int s = warp >> 2;
    const int row = tid & 127;
    const uint32_t trow = tm + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t sc = trow + s_col(s);
    const uint32_t oc = trow + o_col(s);
    const uint64_t sc2 = f32x2(p.scale_log2, p.scale_log2);
    uint32_t nsc = 0, uc = 0;
    bool ok = true;
    for (int u = 0; ok && u < my_units; ++u) {
      const int buf = u % NL;
      if (!(ok = warp_wait(&M.list_full[buf], (u / NL) & 1, abort, lim))) break;
      const UnitList& U = M.L[buf];
      if (U.active[s]) {
        float m = 0.f, l = 0.f;
        bool first = true;
        for (int j = 0; j < U.ns; ++j) {
          const int blk = U.sblk[s][j];
          if (blk == kNoBlock) continue;
          if (!(ok = warp_wait(&M.s_full[s], nsc & 1, abort, lim))) break;
          ++nsc;
          tc_fence_after();
          uint32_t x[128];
          tmem_ld32_at<0>(sc, x);
          tmem_ld32_at<32>(sc + 32, x);
          tmem_ld32_at<64>(sc + 64, x);
          tmem_ld32_at<96>(sc + 96, x);
          tmem_wait_ld();
          if (blk == p.nb - 1) {
            // padded keys of the last block take no part in the softmax
            const int valid = p.N - blk * BN;
#pragma unroll
            for (int c = 0; c < 128; ++c)
              if (c >= valid) x[c] = __float_as_uint(-INFINITY);
          }
          // row max in four independent chains (short dependency latency)
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
          for (int c = 0; c < 128; c += 8) {
            m0 = fmax3(m0, __uint_as_float(x[c]), __uint_as_float(x[c + 1]));
            m1 = fmax3(m1, __uint_as_float(x[c + 2]), __uint_as_float(x[c + 3]));
            m2 = fmax3(m2, __uint_as_float(x[c + 4]), __uint_as_float(x[c + 5]));
            m3 = fmax3(m3, __uint_as_float(x[c + 6]), __uint_as_float(x[c + 7]));
          }
          // lazy rescaling: the exponent base m moves only when the row max
          // exceeds it by more than 2^8 (P then stays <= 256)
          const float mc = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)) * p.scale_log2;
          float alpha = 1.f;
          bool need = false;
          if (first) {
            m = mc;
          } else if (mc > m + kRescaleThreshold) {
            need = true;
            alpha = fast_exp2(m - mc);
            m = mc;
          }
          const uint64_t nm2 = f32x2(-m, -m);
          uint64_t acc2 = f32x2(0.f, 0.f);
          uint32_t lo8[8];  // kLoP: residuals of 16 columns, stored as they complete
#pragma unroll
          for (int c = 0; c < 128; c += 2) {
            float y0, y1;
            f32x2_split(ffma2(f32x2(__uint_as_float(x[c]), __uint_as_float(x[c + 1])), sc2, nm2), y0, y1);
            const float p0 = fast_exp2(y0), p1 = fast_exp2(y1);
            acc2 = fadd2(acc2, f32x2(p0, p1));
            x[c >> 1] = pack_bf16(p0, p1);
            if constexpr (kLoP) {
              // P - bf16(P) over columns [64, 128) of the S buffer (the row is
              // in registers; its tensor-memory copy is no longer read)
              lo8[(c >> 1) & 7] = pack_bf16(p0 - bf16_lo(x[c >> 1]), p1 - bf16_hi(x[c >> 1]));
              if (((c >> 1) & 7) == 7) tmem_st8(sc + Ly::P_OFF + 64 + ((c >> 1) & ~7), lo8);
            }
          }
          // bf16 P over columns [0, 64) of the S buffer (S already read)
          tmem_st32_at<0>(sc + Ly::P_OFF, x);
          tmem_st32_at<32>(sc + Ly::P_OFF + 32, x);
          float s0, s1;
          f32x2_split(acc2, s0, s1);
          l = l * alpha + (s0 + s1);
          first = false;
          if (__any_sync(0xffffffffu, need)) {
            // O holds the previous P.V, complete because that MMA was issued
            // before this S; the next P.V waits for p_full.  (Rare: rolled.)
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
              uint32_t o[32];
              tmem_ld32(oc + c * 32, o);
              tmem_wait_ld();
#pragma unroll
              for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
              tmem_st32(oc + c * 32, o);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&M.p_full[s]);
        }
        if (!ok) break;
        // ---- tile end.  The linear branch is folded into O:
        //   O += rho'_q S_U,  rho'_q = rho_q * g_h * l / (psi_q . z_U),
        // so that the epilogue is out = O / l.  rho'_q (bf16 hi + lo) goes to
        // columns [32, 32 + r) of this slot's S buffer as the A operand of
        // that MMA; q P_h sits in columns [0, r).
        // This code runs once per unit, cold in the instruction cache, so it
        // is written as short rolled loops over 8-column chunks.
        if (!(ok = warp_wait(&M.qt_full[s], uc & 1, abort, lim))) break;
        tc_fence_after();
        const int n = U.a[s] * BM + row;
        const int nn = n < p.N ? n : p.N - 1;
        const int hw = p.Hg * p.W;
        const int pt_ = nn / hw, rem = nn - pt_ * hw;
        const int py = rem / p.W, px = rem - py * p.W;
        if (!(ok = warp_wait(&M.zu_ready[s], uc & 1, abort, lim))) break;
        // pass 1: den = psi_q . z_U
        float den = 0.f;
#pragma unroll 1
        for (int c8 = 0; c8 < R / 8; ++c8) {
          uint32_t v[8];
          tmem_ld8(sc + c8 * 8, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 8; ++e) den = fmaf(phi_fast(__uint_as_float(v[e])), M.zU[s][c8 * 8 + e], den);
        }
        const bool have_o = U.cnt[s] > 0;
        const float lsum = have_o ? l : 1.f;
        const float scale = U.lin_empty[s] ? 0.f : p.gate[U.h] * lsum / den;
        if (p.lse && n < p.N) {
          // statistics a backward pass reads: sum_j exp(s_j / sqrt(d)) = 2^m l
          const size_t ro = ((size_t)U.b * p.H + U.h) * p.N + n;
          p.lse[ro] = have_o ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
          p.den[ro] = U.lin_empty[s] ? __int_as_float(0x7fc00000) : den;
        }
        // pass 2: rho'_q = R(t, y, x) psi_q * scale as bf16 hi + lo
#pragma unroll 1
        for (int c8 = 0; c8 < R / 8; ++c8) {
          uint32_t v[8], rh[4], rl[4];
          tmem_ld8(sc + c8 * 8, v);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int4 rp = M.rope_pair[c8 * 4 + i];
            const float2 c = M.tab[rp.x + (rp.z == 0 ? pt_ : (rp.z == 1 ? py : px)) * rp.y];
            const float x0 = phi_fast(__uint_as_float(v[2 * i])), x1 = phi_fast(__uint_as_float(v[2 * i + 1]));
            const float r0 = (x0 * c.x - x1 * c.y) * scale;
            const float r1 = (x0 * c.y + x1 * c.x) * scale;
            rh[i] = pack_bf16(r0, r1);
            rl[i] = pack_bf16(r0 - bf16_lo(rh[i]), r1 - bf16_hi(rh[i]));
          }
          tmem_st4(sc + 32 + c8 * 4, rh);
          tmem_st4(sc + 32 + R / 2 + c8 * 4, rl);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&M.lin_ready[s]);
        // ---- epilogue: out = O / l
        if (!(ok = warp_wait(&M.l_done[s], uc & 1, abort, lim))) break;
        tc_fence_after();
        const float inv_l = 1.f / lsum;
        const bool write = n < p.N;
        uint4* orow = reinterpret_cast<uint4*>(p.out + (((size_t)U.b * p.N + (write ? n : 0)) * p.H + U.h) * D);
#pragma unroll 1
        for (int c = 0; c < D / 16; ++c) {
          uint32_t o[16];
          tmem_ld16(oc + c * 16, o);
          tmem_wait_ld();
          uint32_t wv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            wv[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv_l, __uint_as_float(o[2 * e + 1]) * inv_l);
          if (write) {
            if (p.out_32b) {
              // one 32-byte store (rows start 256-byte apart from a 32-byte aligned base)
              asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(orow + 2 * c),
                           "r"(wv[0]), "r"(wv[1]), "r"(wv[2]), "r"(wv[3]), "r"(wv[4]), "r"(wv[5]),
                           "r"(wv[6]), "r"(wv[7])
                           : "memory");
            } else {
              orow[2 * c] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
              orow[2 * c + 1] = make_uint4(wv[4], wv[5], wv[6], wv[7]);
            }
            if (p.out_lo) {
              // the bf16 rounding residual of the output (the backward's D needs ~16 bits)
              uint32_t lv[8];
#pragma unroll
              for (int e = 0; e < 8; ++e)
                lv[e] = pack_bf16(__uint_as_float(o[2 * e]) * inv_l - bf16_lo(wv[e]),
                                  __uint_as_float(o[2 * e + 1]) * inv_l - bf16_hi(wv[e]));
              uint4* lrow = reinterpret_cast<uint4*>(p.out_lo + (((size_t)U.b * p.N + n) * p.H + U.h) * D);
              lrow[2 * c] = make_uint4(lv[0], lv[1], lv[2], lv[3]);
              lrow[2 * c + 1] = make_uint4(lv[4], lv[5], lv[6], lv[7]);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&M.o_free[s]);
        ++uc;
      }
      mbar_arrive(&M.list_empty[buf]);
    }
  } else {
    setmaxnreg_dec<136>();
    if (warp >= 10) {
      // ============================================================== P_h, state gather, S_U
      // acc[s] starts as the global state S and loses the state of every
      // block slot s keeps, so it ends as S_U = S - sum_kept S_j; it is then
      // converted in place into the bf16 hi + lo MN-major B operand of the
      // linear-branch MMA (N = d, K = r, 128-byte swizzle).
      const int t = tid - 320;  // 0..63
      constexpr int PER = R * D / 256;  // float4 of a block state per thread
      int pt_head = -1;  // head whose P_h^T the shared-memory operand holds
      float4* accs = reinterpret_cast<float4*>(smem + Ly::acc_off);  // [2][R*D/4]
      uint32_t uc[2] = {0, 0};
      bool ok = true;
      for (int u = 0; ok && u < my_units; ++u) {
        const int buf = u % NL;
        if (!(ok = warp_wait(&M.list_full[buf], (u / NL) & 1, abort, lim))) break;
        const UnitList& U = M.L[buf];
        const int b = U.b, h = U.h;
        const size_t bh = (size_t)b * p.H + h;
        // The global state, where both accumulators start, is requested
        // before the wait below so that its latency hides behind it.  Thread t
        // owns accumulator slots t + 64 i (float4, i < PER) of both slots'
        // accumulators; slot i holds the four state elements at
        // 8 (t + 64 (i / 2)) + 4 (i % 2), so that a state is read with 32-byte
        // loads (two slots each) while the shared-memory slots stay contiguous
        // across the warp.
        float4 g4[PER];
#pragma unroll
        for (int i2 = 0; i2 < PER / 2; ++i2)
          ldg_na8(p.S_glb + bh * R * D + 8 * (t + 64 * i2), g4[2 * i2], g4[2 * i2 + 1]);
        // the previous unit's linear-branch MMAs read these accumulators
        // (and its q P_h MMAs read P_h^T) -- wait for them
#pragma unroll
        for (int s = 0; s < 2; ++s)
          if (ok && uc[s] >= 1) ok = warp_wait(&M.l_done[s], (uc[s] - 1) & 1, abort, lim);
        if (!ok) break;
        // P_h^T (K-major, N = r rows, K = d, 128-byte swizzle), rewritten only
        // when the head changes; P_h is read 8 values (16 bytes) at a time
        {
          if (h != pt_head) {
            uint8_t* pt = smem + Ly::pt_off;
            for (int e8 = t; e8 < R * D / 8; e8 += 64) {
              const int c = e8 / (R / 8), r0 = (e8 % (R / 8)) * 8;
              const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.P + ((size_t)h * D + c) * R + r0));
              const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
              const int byte = (c & 63) * 2;
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                const int rr = r0 + j;
                const int chunk = (byte >> 4) ^ (rr & 7);
                *reinterpret_cast<uint16_t*>(pt + (c >> 6) * (32 * 128) + rr * 128 + chunk * 16 + (byte & 15)) =
                    (uint16_t)(wv[j >> 1] >> (16 * (j & 1)));
              }
            }
            fence_proxy_async_smem();
            pt_head = h;
          }
          mbar_arrive(&M.pt_full);
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) {
          accs[t + 64 * i] = g4[i];
          accs[R * D / 4 + t + 64 * i] = g4[i];
        }
        const float zg = t < R ? p.z_glb[bh * R + t] : 0.f;
        float zs[2] = {zg, zg};
        for (int j = 0; j < U.nu; ++j) {
          const size_t st = bh * p.nb + U.ulist[j];
          const float4* src = reinterpret_cast<const float4*>(p.S_blk + st * R * D);
          const int mk = U.umask[j];
          float4 xv[PER];
#pragma unroll
          for (int i2 = 0; i2 < PER / 2; ++i2)
            ldg_na8(reinterpret_cast<const float*>(src) + 8 * (t + 64 * i2), xv[2 * i2], xv[2 * i2 + 1]);
          const float zv = t < R ? __ldg(p.z_blk + st * R + t) : 0.f;
#pragma unroll
          for (int sl = 0; sl < 2; ++sl) {
            if (!((mk >> sl) & 1)) continue;
            float4* a = accs + sl * (R * D / 4);
#pragma unroll
            for (int i = 0; i < PER; ++i) {
              // packed f32x2 subtractions: half the instructions
              const float4 v = a[t + 64 * i];
              float r0, r1, r2, r3;
              f32x2_split(fsub2(f32x2(v.x, v.y), f32x2(xv[i].x, xv[i].y)), r0, r1);
              f32x2_split(fsub2(f32x2(v.z, v.w), f32x2(xv[i].z, xv[i].w)), r2, r3);
              a[t + 64 * i] = make_float4(r0, r1, r2, r3);
            }
            zs[sl] -= zv;
          }
        }
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (!ok || !U.active[s]) continue;
          float4* a = accs + s * (R * D / 4);
          float4 v[PER];
#pragma unroll
          for (int i = 0; i < PER; ++i) v[i] = a[t + 64 * i];
          // every thread has read its part before anyone overwrites the region
          mbar_arrive(&M.cvt[s]);
          if (!(ok = warp_wait(&M.cvt[s], uc[s] & 1, abort, lim))) continue;
          uint8_t* su_hi = reinterpret_cast<uint8_t*>(a);
          uint8_t* su_lo = su_hi + Ly::SU_BYTES;
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            const uint32_t h01 = pack_bf16(v[i].x, v[i].y), h23 = pack_bf16(v[i].z, v[i].w);
            const uint32_t l01 = pack_bf16(v[i].x - bf16_lo(h01), v[i].y - bf16_hi(h01));
            const uint32_t l23 = pack_bf16(v[i].z - bf16_lo(h23), v[i].w - bf16_hi(h23));
            const int f = 8 * (t + 64 * (i >> 1)) + 4 * (i & 1);
            const int c = f / D, e = f % D;
            const uint32_t off = (e >> 6) * (R * 128) + (c >> 3) * 1024 + (c & 7) * 128 +
                                 ((((e & 63) >> 3) ^ (c & 7)) << 4) + (e & 7) * 2;
            *reinterpret_cast<uint2*>(su_hi + off) = make_uint2(h01, h23);
            *reinterpret_cast<uint2*>(su_lo + off) = make_uint2(l01, l23);
          }
          if (t < R) M.zU[s][t] = zs[s];
          fence_proxy_async_smem();
          mbar_arrive(&M.zu_ready[s]);
          ++uc[s];
        }
        if (!ok) break;
        mbar_arrive(&M.list_empty[buf]);
      }
    } else if (warp == 8) {
      // ================================================================ producer
      uint32_t g = 0, uc[2] = {0, 0};
      int ring_par[NR], q_par[2] = {-1, -1};
      for (int i = 0; i < NR; ++i) ring_par[i] = -1;
      bool ok = true;
      if (lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
      }
      // Unit list of unit u into buffer u % NL, by the whole warp: both kept
      // lists are validated (in range, above the previous entry of the row;
      // a bad entry is skipped and reported), marked in one bitmap per slot
      // and read back as one ascending union with a per-slot mask, and as the
      // steps: the n_sh blocks both slots keep and the n_sp = min(n_0, n_1)
      // pairs of slot-only blocks alternate (shared, pair, shared, pair, ...,
      // then the rest of the longer kind), and the slot-only blocks left over
      // when n_0 != n_1 (a skipped bad entry, or an idle second slot) follow
      // as single-slot steps.
      auto build_list = [&](int u) -> bool {
        const int buf = u % NL;
        if (u >= NL && !warp_wait(&M.list_empty[buf], ((u / NL) - 1) & 1, abort, lim)) return false;
        UnitList& U = M.L[buf];
        int b, h, pair;
        decode_unit(p, (int)blockIdx.x + u * (int)gridDim.x, b, h, pair);
        const int a0 = 2 * pair, a1 = 2 * pair + 1;
        const size_t bh = (size_t)b * p.H + h;
        M.kept_bits[0][lane] = 0u;
        M.kept_bits[1][lane] = 0u;
        __syncwarp();
        int err = 0;
        int kbh = p.kb;  // this head's kept count (a count outside [1, kb] is clamped and reported)
        if (p.kb_h) {
          const int want = p.kb_h[h];
          kbh = min(max(want, 1), p.kb);
          err = kbh != want;
        }
        for (int i = lane; i < 2 * kbh; i += 32) {
          const int sl = i >= kbh ? 1 : 0, e = i - sl * kbh, a = sl ? a1 : a0;
          if (a >= p.nb) continue;
          const int32_t* row = p.idx + (bh * p.nb + a) * p.kb;
          const int v = row[e];
          if (v >= 0 && v < p.nb && (e == 0 || v > row[e - 1]))
            atomicOr(&M.kept_bits[sl][v >> 5], 1u << (v & 31));
          else
            err = 1;
        }
        __syncwarp();
        const uint32_t m0 = M.kept_bits[0][lane], m1 = M.kept_bits[1][lane], mu = m0 | m1;
        const uint32_t sh = m0 & m1, x0 = m0 & ~m1, x1 = m1 & ~m0;
        // inclusive prefix counts over lanes (lane w holds blocks [32 w, 32 w + 32)),
        // two 16-bit counts per word: union | shared << 16, slot-0-only | slot-1-only << 16
        int pa = __popc(mu) | (__popc(sh) << 16), pb = __popc(x0) | (__popc(x1) << 16);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int ta = __shfl_up_sync(0xffffffffu, pa, off), tb = __shfl_up_sync(0xffffffffu, pb, off);
          if (lane >= off) {
            pa += ta;
            pb += tb;
          }
        }
        const int ta = __shfl_sync(0xffffffffu, pa, 31), tb = __shfl_sync(0xffffffffu, pb, 31);
        const int nu = ta & 0xffff, nsh = ta >> 16, n0 = tb & 0xffff, n1 = tb >> 16;
        const int nsp = min(n0, n1), mlt = min(nsh, nsp);
        int pos = (pa & 0xffff) - __popc(mu);
        for (uint32_t rem = mu; rem; rem &= rem - 1) {
          const int bit = __ffs(rem) - 1;
          U.ulist[pos] = (uint16_t)(lane * 32 + bit);
          U.umask[pos] = (uint8_t)(((m0 >> bit) & 1u) | (((m1 >> bit) & 1u) << 1));
          ++pos;
        }
        int i = (pa >> 16) - __popc(sh);  // shared block i -> step 2 i, or 2 mlt + (i - mlt)
        for (uint32_t rem = sh; rem; rem &= rem - 1, ++i) {
          const int st = i < mlt ? 2 * i : 2 * mlt + (i - mlt);
          U.sblk[0][st] = U.sblk[1][st] = (uint16_t)(lane * 32 + __ffs(rem) - 1);
        }
        // slot-only block k of slot sl: pair k -> step 2 k + 1, or 2 mlt + (k - mlt);
        // leftovers after the pairs -> single-slot steps after nsh + nsp
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          int k = sl ? (pb >> 16) - __popc(x1) : (pb & 0xffff) - __popc(x0);
          for (uint32_t rem = sl ? x1 : x0; rem; rem &= rem - 1, ++k) {
            const uint16_t blk = (uint16_t)(lane * 32 + __ffs(rem) - 1);
            if (k < nsp) {
              U.sblk[sl][k < mlt ? 2 * k + 1 : 2 * mlt + (k - mlt)] = blk;
            } else {
              const int st = nsh + nsp + (sl ? n0 - nsp : 0) + (k - nsp);
              U.sblk[sl][st] = blk;
              U.sblk[sl ^ 1][st] = kNoBlock;
            }
          }
        }
        const int c0 = nsh + n0, c1 = nsh + n1;
        if (__any_sync(0xffffffffu, err) && lane == 0) M.err = 1;
        if (lane == 0) {
          U.b = b;
          U.h = h;
          U.a[0] = a0;
          U.a[1] = a1;
          U.active[0] = a0 < p.nb;
          U.active[1] = a1 < p.nb;
          U.nu = nu;
          U.ns = nsh + max(n0, n1);
          U.cnt[0] = c0;
          U.cnt[1] = c1;
          U.lin_empty[0] = c0 >= p.nb;
          U.lin_empty[1] = c1 >= p.nb;
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) mbar_arrive(&M.list_full[buf]);
        return true;
      };
      if (my_units > 0) ok = build_list(0);
      for (int u = 0; ok && u < my_units; ++u) {
        const UnitList& U = M.L[u % NL];
        const int ns = U.ns, b = U.b, h = U.h;
        // one K or V tile of a key block into the next ring slot, by block index
        auto load_tile = [&](const CUtensorMap* mp, int blk) -> bool {
          const int slot = g % NR;
          if (g >= (uint32_t)NR && !mbar_wait(&M.ring_empty[slot], ((g / NR) - 1) & 1, abort, lim)) return false;
          mbar_expect_tx(&M.ring_full[slot], TILE);
          for (int ka = 0; ka < 2; ++ka)
            tma_load_4d(smem + Ly::ring_off + slot * TILE + ka * (BN * 128), mp, &M.ring_full[slot], ka * 64,
                        h, blk * BN, b);
          ring_par[slot] = (g / NR) & 1;
          ++g;
          return true;
        };
        // the tiles of step j in the order the MMAs first use them: K then V of
        // a shared or single-slot step; K_0, K_1, V_0, V_1 of a paired step.
        // part 0 is the first two tiles, part 1 the rest (a pair's V tiles).
        auto load_step = [&](int j, int part) -> bool {
          const int b0 = U.sblk[0][j], b1 = U.sblk[1][j];
          if (b0 != kNoBlock && b1 != kNoBlock && b0 != b1)
            return part == 0 ? load_tile(&tmK, b0) && load_tile(&tmK, b1)
                             : load_tile(&tmV, b0) && load_tile(&tmV, b1);
          const int blk = b0 != kNoBlock ? b0 : b1;
          return part == 0 ? load_tile(&tmK, blk) && load_tile(&tmV, blk) : true;
        };
        // the first two tiles of the first step, then the Q tiles (after the
        // previous unit's last S MMA has read them), so that the first copies
        // overlap the previous unit's tail, then the rest of the first step.
        // The ring holds three tiles: a pair's fourth tile goes into the slot
        // its first tile (K_0) frees, which needs the unit's first S MMA and
        // so its Q tile -- Q goes out before it.
        if (lane == 0) {
          if (ns > 0) ok = load_step(0, 0);
          for (int sl = 0; sl < 2 && ok; ++sl) {
            if (!U.active[sl]) continue;
            if (uc[sl] >= 1 && !(ok = mbar_wait(&M.q_empty[sl], (uc[sl] - 1) & 1, abort, lim))) break;
            mbar_expect_tx(&M.q_full[sl], TILE);
            for (int ka = 0; ka < 2; ++ka)
              tma_load_4d(smem + Ly::q_off + sl * TILE + ka * (BM * 128), &tmQ, &M.q_full[sl], ka * 64, h,
                          U.a[sl] * BM, b);
            q_par[sl] = uc[sl] & 1;
            ++uc[sl];
          }
          if (ok && ns > 0) ok = load_step(0, 1);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        // the next unit's list while this unit's copies are in flight
        if (ok && u + 1 < my_units) ok = build_list(u + 1);
        if (lane == 0)
          for (int j = 1; ok && j < ns; ++j) ok = load_step(j, 0) && load_step(j, 1);
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        __syncwarp();
      }
      // Drain: copies complete on their own; wait (bounded) for the last ones.
      if (lane == 0) {
        int no_abort = 0;
        for (int i = 0; i < NR; ++i)
          if (ring_par[i] >= 0) mbar_wait(&M.ring_full[i], ring_par[i], &no_abort);
        for (int i = 0; i < 2; ++i)
          if (q_par[i] >= 0) mbar_wait(&M.q_full[i], q_par[i], &no_abort);
        if (no_abort) *abort = 1;
      }
    } else if (warp == 9 && lane == 0) {
      // ================================================================ MMA issuer
      constexpr uint32_t idesc_s = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, BN);
      constexpr uint32_t idesc_pv = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, D);
      constexpr uint32_t idesc_qt = instr_desc(kFmtBF16, kFmtBF16, false, false, 128, R);
      constexpr uint32_t idesc_l = instr_desc(kFmtBF16, kFmtBF16, false, true, 128, D);
      const uint32_t sQ = smem_u32(smem + Ly::q_off);
      const uint32_t sR = smem_u32(smem + Ly::ring_off);
      const uint32_t sPT = smem_u32(smem + Ly::pt_off);
      const uint32_t sAcc = smem_u32(smem + Ly::acc_off);
      // k-step-0 descriptors of the Q tiles, of the ring slots as K
      // (K-major) and as V (MN-major), all with 128-byte swizzle
      // (a tile further on is TILE / 16 more in the start-address field)
      const uint64_t dq0[2] = {desc_k_sw128(sQ, BM, 0), desc_k_sw128(sQ + TILE, BM, 0)};
      const uint64_t dr_base = desc_k_sw128(sR, BN, 0);
      const uint64_t dv_base = smem_desc(sR, BN * 128, 1024, kSwizzle128B);
      uint32_t g = 0, np[2] = {0, 0}, uc[2] = {0, 0};

      bool ok = true;
      for (int u = 0; ok && u < my_units; ++u) {
        const int buf = u % NL;
        if (!(ok = mbar_wait(&M.list_full[buf], (u / NL) & 1, abort, lim))) break;
        const UnitList& U = M.L[buf];
#pragma unroll
        for (int s = 0; s < 2; ++s)
          if (ok && U.active[s]) ok = mbar_wait(&M.q_full[s], uc[s] & 1, abort, lim);
        if (!ok) break;
        int pend_v[2] = {-1, -1};  // ring index of the V tile a slot's next P.V uses
        // A ring tile is released by the last MMA that reads it.  Within a
        // step slot 0's MMAs go out before slot 1's (S here, P.V in the next
        // step or at the tile end), so a tile both slots read is released by
        // slot 1's MMA, and a tile one slot reads by that slot's.
        bool rel_v[2] = {false, false};
        bool first_pv[2] = {true, true};
        auto issue_pv = [&](int s) -> bool {
          if (!mbar_wait(&M.p_full[s], np[s] & 1, abort, lim)) return false;
          // the previous unit's epilogue must have read O first
          if (first_pv[s] && uc[s] >= 1 && !mbar_wait(&M.o_free[s], (uc[s] - 1) & 1, abort, lim)) return false;
          ++np[s];
          const uint32_t gv = (uint32_t)pend_v[s];
          if (!mbar_wait(&M.ring_full[gv % NR], (gv / NR) & 1, abort, lim)) return false;
          tc_fence_after();
          const uint64_t dv = dv_base + (uint64_t)(gv % NR) * (TILE >> 4);
          const uint32_t acc0 = first_pv[s] ? 0u : 1u;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            mma_ts(tm + o_col(s), tm + s_col(s) + Ly::P_OFF + kk * 8, dv + (uint64_t)(kk * 16 * 128 >> 4),
                   idesc_pv, kk == 0 ? acc0 : 1u);
            if constexpr (kLoP)
              mma_ts(tm + o_col(s), tm + s_col(s) + Ly::P_OFF + 64 + kk * 8, dv + (uint64_t)(kk * 16 * 128 >> 4),
                     idesc_pv, 1u);
          }
          first_pv[s] = false;
          if (rel_v[s]) mma_commit(&M.ring_empty[gv % NR]);
          pend_v[s] = -1;
          return true;
        };
        for (int j = 0; ok && j < U.ns; ++j) {
          // the step's tiles in the producer's order: K, V (one block, used by
          // every slot working in the step) or K_0, K_1, V_0, V_1 (a pair)
          const int blk[2] = {U.sblk[0][j], U.sblk[1][j]};
          const bool paired = blk[0] != kNoBlock && blk[1] != kNoBlock && blk[0] != blk[1];
          // the one reader (paired step or idle slot) or slot 1 releases
          const bool last[2] = {paired || blk[1] == kNoBlock, true};
          uint32_t gk[2], gv[2];
          if (paired) {
            gk[0] = g;
            gk[1] = g + 1;
            gv[0] = g + 2;
            gv[1] = g + 3;
            g += 4;
          } else {
            gk[0] = gk[1] = g;
            gv[0] = gv[1] = g + 1;
            g += 2;
          }
          // slot 0's pending P.V needs no new tile: it goes out before the
          // wait for K, which frees its V slot for the copies sooner.  Every
          // pending P.V goes out in this step, also for a slot idle in it: a
          // deferred P.V would pin its V tile in the ring.
#pragma unroll
          for (int s = 0; s < 2; ++s) {
            if (ok && pend_v[s] >= 0) ok = issue_pv(s);
            if (!ok || blk[s] == kNoBlock) continue;
            const uint32_t k = gk[s];
            if (!(ok = mbar_wait(&M.ring_full[k % NR], (k / NR) & 1, abort, lim))) break;
            tc_fence_after();
            const uint64_t dq = dq0[s], dk = dr_base + (uint64_t)(k % NR) * (TILE >> 4);
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tm + s_col(s), dq + kstep_k_sw128(BM, kk), dk + kstep_k_sw128(BN, kk), idesc_s,
                     kk > 0 ? 1u : 0u);
            mma_commit(&M.s_full[s]);
            if (last[s]) mma_commit(&M.ring_empty[k % NR]);
            pend_v[s] = (int)gv[s];
            rel_v[s] = last[s];
          }
        }
        // tile end, per slot as soon as its last P.V is out: q P_h into the
        // (now free) S columns; Q is then free for the next unit.  Then
        // O += rho'_q S_U with rho'_q read from tensor memory (written by the
        // softmax warps) and S_U from the gather.
        if (!(ok = mbar_wait(&M.pt_full, u & 1, abort, lim))) break;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (ok && pend_v[s] >= 0) ok = issue_pv(s);
          if (!ok || !U.active[s]) continue;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tm + s_col(s), dq0[s] + kstep_k_sw128(BM, kk), desc_k_sw128(sPT, 32, kk), idesc_qt,
                   kk > 0 ? 1u : 0u);
          mma_commit(&M.qt_full[s]);
          mma_commit(&M.q_empty[s]);
        }
        if (!ok) break;
#pragma unroll
        for (int s = 0; s < 2; ++s) {
          if (!ok || !U.active[s]) continue;
          if (!(ok = mbar_wait(&M.lin_ready[s], uc[s] & 1, abort, lim))) continue;
          if (!(ok = mbar_wait(&M.zu_ready[s], uc[s] & 1, abort, lim))) continue;
          tc_fence_after();
          const uint32_t suh = sAcc + s * (R * D * 4), sul = suh + Ly::SU_BYTES;
          const uint32_t a_hi = tm + s_col(s) + 32, a_lo = a_hi + R / 2;
#pragma unroll
          for (int kk = 0; kk < R / 16; ++kk) {
            const uint64_t bh_ = smem_desc(suh + kk * 2048, R * 128, 1024, kSwizzle128B);
            const uint64_t bl_ = smem_desc(sul + kk * 2048, R * 128, 1024, kSwizzle128B);
            // a slot without any kept block has no P.V in O yet
            mma_ts(tm + o_col(s), a_hi + kk * 8, bh_, idesc_l, (kk == 0 && U.cnt[s] == 0) ? 0u : 1u);
            mma_ts(tm + o_col(s), a_hi + kk * 8, bl_, idesc_l, 1u);
            mma_ts(tm + o_col(s), a_lo + kk * 8, bh_, idesc_l, 1u);
          }
          mma_commit(&M.l_done[s]);
          ++uc[s];
        }
        if (!ok) break;
        mbar_arrive(&M.list_empty[buf]);
      }
      mma_commit(&M.mma_final);
      int no_abort = 0;
      mbar_wait(&M.mma_final, 0, &no_abort);
      if (no_abort) *abort = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tm, 512);
  }
  if (tid == 0 && p.dev_err && (M.abort || M.err))
    atomicOr(p.dev_err, (M.abort ? ROLA_DEVERR_TIMEOUT : 0) | (M.err ? ROLA_DEVERR_BAD_INDEX : 0));
}

template <int R>
static rola_status_t launch(const rola_shape_t* s, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                            Params prm, cudaStream_t cs) {
  using Ly = Layout<R>;
  CUtensorMap mq, mk, mv;
  if (!rola_host::make_act_map(&mq, q, s, 128) || !rola_host::make_act_map(&mk, k, s, 128) ||
      !rola_host::make_act_map(&mv, v, s, 128))
    return ROLA_ERR_CUDA;
  const size_t smem = Ly::misc_off + sizeof(Misc) + 1024;
  auto kern = prm.out_lo ? rola_attn_pair_kernel<R, true> : rola_attn_pair_kernel<R, false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return ROLA_ERR_CUDA;
  const int nsm = rola_host::sm_count();
  const int grid = prm.units < nsm ? prm.units : nsm;
  kern<<<grid, kThreads, smem, cs>>>(mq, mk, mv, prm);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

}  // namespace pairk

// Used by rola_attention_fwd for d = 128, 128-token blocks, k_b <= 256 and a
// latent grid whose rotary table fits in shared memory.
bool pair_kernel_supports(const rola_shape_t* s) {
  if (!(s->d == 128 && s->block == 128 && s->k_b <= pairk::kMaxKept && (s->r == 16 || s->r == 32)))
    return false;
  if (rola_num_blocks(s) > pairk::kMaxBlocks) return false;
  const int rh = 2 * (s->r / 6), rt = s->r - 2 * rh;
  const long long entries = (long long)s->T * (rt / 2) + (long long)(s->Hg + s->W) * (rh / 2);
  return entries <= pairk::kTabCap;
}

rola_status_t launch_pair_kernel(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                 const float* S_blk, const float* z_blk, const float* S_glb,
                                 const float* z_glb, const float* gate, uint16_t* out, int32_t* dev_err,
                                 const int32_t* kb_h, uint64_t wait_ns, float* lse, float* den,
                                 uint16_t* out_lo, cudaStream_t cs) {
  pairk::Params prm{};
  prm.wait_ns = wait_ns;
  prm.kb_h = kb_h;
  prm.lse = lse;
  prm.den = den;
  prm.out_lo = out_lo;
  prm.B = s->B;
  prm.H = s->H;
  prm.N = s->N;
  prm.nb = rola_num_blocks(s);
  prm.kb = s->k_b;
  prm.T = s->T;
  prm.Hg = s->Hg;
  prm.W = s->W;
  prm.npairs = (prm.nb + 1) / 2;
  prm.units = s->B * s->H * prm.npairs;
  prm.scale_log2 = (float)(1.4426950408889634 / sqrt((double)s->d));
  prm.idx = idx;
  prm.P = P;
  prm.S_blk = S_blk;
  prm.z_blk = z_blk;
  prm.S_glb = S_glb;
  prm.z_glb = z_glb;
  prm.gate = gate;
  prm.out = out;
  prm.out_32b = rola_host::aligned(out, 32) ? 1 : 0;
  prm.dev_err = dev_err;
  rola_host::rope_frequencies(s->r, s->rope_base, prm.rope.freq, prm.rope.axis);
  {
    rola_host::RopeTabLayout tl;
    rola_host::rope_table_layout(s, prm.rope.axis, &tl);
    for (int i = 0; i < 16; ++i) {
      prm.tab_base[i] = tl.base[i];
      prm.tab_stride[i] = tl.stride[i];
    }
    for (int i = 0; i < 17; ++i) prm.tab_first[i] = tl.first[i];
    prm.tab_entries = tl.entries;
  }
  if (s->r == 32) return pairk::launch<32>(s, q, k, v, prm, cs);
  return pairk::launch<16>(s, q, k, v, prm, cs);
}

}  // namespace rola
