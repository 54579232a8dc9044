// Block selector: mean-pool q and k per block (float64, exact block sums of
// bf16), score every query block against every key block with the float64
// tensor-core path (DMMA m8n8k4), and keep the top k_b key blocks per query
// block by (-score, index), emitted ascending.
//
// SparkDiffusion write-up (0539edu.com news page), section 01: sparse
// attention keeps only the important query-key blocks; section 05: RoLA's
// sparse branch keeps the high-energy query-key block interactions.  The
// mean-pooled score is this library's concrete selector (the pages give none).
#include <float.h>
#include <math.h>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola {

// ---------------------------------------------------------------- pooling
// grid (n_blocks, B, 2 [q or k]), 256 threads; each thread owns 8 adjacent
// bf16 columns of the [N, H*d] token rows and sums the block's valid tokens.
__global__ void __launch_bounds__(256) pool_kernel(const uint16_t* __restrict__ q,
                                                   const uint16_t* __restrict__ k,
                                                   double* __restrict__ qbar,
                                                   double* __restrict__ kbar, int N, int H, int d,
                                                   int bs, int nb) {
  const int blk = blockIdx.x, b = blockIdx.y;
  const uint16_t* src = blockIdx.z == 0 ? q : k;
  double* dst = blockIdx.z == 0 ? qbar : kbar;
  const int HD = H * d;
  const int n0 = blk * bs, n1 = min(N, n0 + bs);
  const double cnt = (double)(n1 - n0);
  const size_t row_stride = (size_t)HD / 8;  // in uint4
  for (int c8 = threadIdx.x; c8 < HD / 8; c8 += blockDim.x) {
    double acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0;
    const uint4* p = reinterpret_cast<const uint4*>(src + ((size_t)b * N + n0) * HD) + c8;
    int n = n0;
    for (; n + 8 <= n1; n += 8) {
      uint4 u[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) u[t] = __ldg(p + (size_t)t * row_stride);
      p += 8 * row_stride;
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const uint32_t w[4] = {u[t].x, u[t].y, u[t].z, u[t].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += (double)bf16_lo(w[i]);
          acc[2 * i + 1] += (double)bf16_hi(w[i]);
        }
      }
    }
    for (; n < n1; ++n) {
      const uint4 u = __ldg(p);
      p += row_stride;
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[2 * i] += (double)bf16_lo(w[i]);
        acc[2 * i + 1] += (double)bf16_hi(w[i]);
      }
    }
    const int col = c8 * 8, h = col / d, c = col % d;
    double* o = dst + (((size_t)b * H + h) * nb + blk) * d + c;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = acc[i] / cnt;
  }
}

// ---------------------------------------------------------------- scores
// sigma[b,h,a,j] = qbar[b,h,a,:] . kbar[b,h,j,:] / sqrt(d) in float64.
// CTA tile 64 x 64 (4 warps of 32 x 32); d is staged through shared memory in
// chunks of 32 by asynchronous copies (cp.async, two stages: the next chunk
// lands while the DMMA m8n8k4 tiles run on the current one); rows past
// n_blocks are zero-filled by the copy.
constexpr int kScTile = 64, kScChunk = 32, kScStride = 36;  // stride keeps DMMA loads conflict-free
constexpr int kScStageDoubles = 2 * kScTile * kScStride;     // A and B chunk of one stage
constexpr size_t kScSmemBytes = 2 * kScStageDoubles * sizeof(double);

ROLA_DEV void dmma_8x8x4(double (&c)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(c[0]), "+d"(c[1])
               : "d"(a), "d"(b));
}
// 16-byte asynchronous global -> shared copy; src_bytes = 0 writes zeros.
ROLA_DEV void cp_async16(void* dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
               : "memory");
}
ROLA_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
ROLA_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(128) score_kernel(const double* __restrict__ qbar,
                                                    const double* __restrict__ kbar,
                                                    double* __restrict__ sigma, int H, int d,
                                                    int nb) {
  extern __shared__ double sc_smem[];  // [2 stages][A | B][kScTile * kScStride]
  const int bh = blockIdx.z;
  const int row0 = blockIdx.y * kScTile, col0 = blockIdx.x * kScTile;
  const double* A = qbar + (size_t)bh * nb * d;
  const double* Bm = kbar + (size_t)bh * nb * d;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wr = (warp >> 1) * 32, wc = (warp & 1) * 32;
  // chunk c0 of both operands into stage st: 64 rows x 16 pieces of 16 bytes each
  auto load = [&](int st, int c0) {
    double* sA = sc_smem + st * kScStageDoubles;
    double* sB = sA + kScTile * kScStride;
    for (int e = threadIdx.x; e < kScTile * (kScChunk / 2); e += blockDim.x) {
      const int r = e / (kScChunk / 2), c = (e % (kScChunk / 2)) * 2;
      const bool ra = row0 + r < nb, rb = col0 + r < nb;
      cp_async16(sA + r * kScStride + c, ra ? A + (size_t)(row0 + r) * d + c0 + c : A, ra ? 16u : 0u);
      cp_async16(sB + r * kScStride + c, rb ? Bm + (size_t)(col0 + r) * d + c0 + c : Bm, rb ? 16u : 0u);
    }
    cp_async_commit();
  };
  double acc[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

  const int nchunks = d / kScChunk;
  load(0, 0);
  for (int ch = 0; ch < nchunks; ++ch) {
    if (ch + 1 < nchunks) {
      load((ch + 1) & 1, (ch + 1) * kScChunk);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const double* sA = sc_smem + (ch & 1) * kScStageDoubles;
    const double* sB = sA + kScTile * kScStride;
#pragma unroll
    for (int kk = 0; kk < kScChunk; kk += 4) {
      double af[4], bf[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        af[i] = sA[(wr + 8 * i + (lane >> 2)) * kScStride + kk + (lane & 3)];
        bf[i] = sB[(wc + 8 * i + (lane >> 2)) * kScStride + kk + (lane & 3)];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_8x8x4(acc[i][j], af[i], bf[j]);
    }
    __syncthreads();  // stage (ch & 1) is refilled by the load two chunks on
  }
  const double rs = sqrt((double)d);
  double* S = sigma + (size_t)bh * nb * nb;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = row0 + wr + 8 * i + (lane >> 2);
      const int c = col0 + wc + 8 * j + 2 * (lane & 3);
      if (r < nb) {
        if (c < nb) S[(size_t)r * nb + c] = acc[i][j][0] / rs;
        if (c + 1 < nb) S[(size_t)r * nb + c + 1] = acc[i][j][1] / rs;
      }
    }
}

// ---------------------------------------------------------------- top-k
// One warp per (b, h, query block).  Lane l holds the scores of blocks l,
// l + 32, ... (MAXP per lane, n_blocks <= 32 * MAXP).  Order: score
// descending, then block index ascending.  A row keeps kb blocks, or
// kb_h[h] of them when per-head counts are given (the row stride stays kb;
// entries past the head's count are set to -1; a count outside [1, kb] is
// clamped into it and reported as ROLA_DEVERR_BAD_INDEX).
//
// Fast path (k_b <= 32, k_b < n_blocks): the k_b-th largest of the 32 lane
// maxima, T, is a lower bound of the k_b-th largest score (k_b lanes hold a
// score >= T), so the kept set lies among the scores >= T.  Those candidates
// (typically a few dozen) go to shared memory and each one's exact rank is
// counted against the others; rank < k_b is kept.  With more than kCandCap
// candidates, or a larger k_b, the warp falls back to k_b rounds of a warp
// arg-max.  The kept set is written in ascending block order.
constexpr int kMaxPerLane = 32;
constexpr int kCandCap = 256;
constexpr int kTopkWarps = 8;

template <int MAXP>
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const double* __restrict__ sigma,
                                                               int32_t* __restrict__ idx, int rows,
                                                               int nb, int kb_max,
                                                               const int32_t* __restrict__ kb_h, int H,
                                                               int32_t* dev_err) {
  __shared__ double cand_v[kTopkWarps][kCandCap];
  __shared__ int cand_j[kTopkWarps][kCandCap];
  __shared__ uint32_t kept_bits[kTopkWarps][32];
  const int wib = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int warp = blockIdx.x * kTopkWarps + wib;
  if (warp >= rows) return;  // uniform per warp
  const double* s = sigma + (size_t)warp * nb;
  int32_t* out = idx + (size_t)warp * kb_max;
  int kb = kb_max;
  if (kb_h) {
    const int want = kb_h[(warp / nb) % H];
    kb = min(max(want, 1), kb_max);
    if (kb != want && lane == 0 && dev_err) atomicOr(dev_err, ROLA_DEVERR_BAD_INDEX);
    for (int e = kb + lane; e < kb_max; e += 32) out[e] = -1;
  }
  double v[MAXP];
#pragma unroll
  for (int i = 0; i < MAXP; ++i) {
    const int j = i * 32 + lane;
    v[i] = j < nb ? s[j] : -INFINITY;
  }
  constexpr int kNone = 0x7fffffff;
  uint32_t taken = 0;
  bool done = false;
  if (kb >= nb) {
    taken = 0xffffffffu;
    done = true;
  } else if (kb <= 32) {
    double m = v[0];
#pragma unroll
    for (int i = 1; i < MAXP; ++i) m = fmax(m, v[i]);
    // rank of this lane's maximum among the 32 (value desc, lane asc)
    int rank = 0;
#pragma unroll
    for (int l2 = 0; l2 < 32; ++l2) {
      const double o = __shfl_sync(0xffffffffu, m, l2);
      rank += (o > m || (o == m && l2 < lane)) ? 1 : 0;
    }
    const uint32_t who = __ballot_sync(0xffffffffu, rank == kb - 1);
    const double T = __shfl_sync(0xffffffffu, m, __ffs(who) - 1);
    // gather the candidates (finite: at least k_b lanes hold a real score)
    int C = 0;
    const uint32_t below = (1u << lane) - 1u;
#pragma unroll
    for (int i = 0; i < MAXP; ++i) {
      const int j = i * 32 + lane;
      const bool c = j < nb && v[i] >= T;
      const uint32_t ball = __ballot_sync(0xffffffffu, c);
      if (c) {
        const int pos = C + __popc(ball & below);
        if (pos < kCandCap) {
          cand_v[wib][pos] = v[i];
          cand_j[wib][pos] = j;
        }
      }
      C += __popc(ball);
    }
    kept_bits[wib][lane] = 0;
    __syncwarp();
    if (C <= kCandCap) {
      for (int c = lane; c < C; c += 32) {
        const double sv = cand_v[wib][c];
        const int sj = cand_j[wib][c];
        int r = 0;
        for (int c2 = 0; c2 < C; ++c2) {
          const double o = cand_v[wib][c2];
          r += (o > sv || (o == sv && cand_j[wib][c2] < sj)) ? 1 : 0;
        }
        if (r < kb) atomicOr(&kept_bits[wib][sj >> 5], 1u << (sj & 31));
      }
      __syncwarp();
#pragma unroll
      for (int i = 0; i < MAXP; ++i) taken |= ((kept_bits[wib][i] >> lane) & 1u) << i;
      done = true;
    }
  }
  if (!done) {
    // k_b rounds of a warp arg-max; only the lane that owned the winner
    // looks for its next candidate
    auto local_best = [&](double& best, int& bidx) {
      best = -INFINITY;
      bidx = kNone;
#pragma unroll
      for (int i = 0; i < MAXP; ++i) {
        const int j = i * 32 + lane;
        if (j < nb && !((taken >> i) & 1u) && (bidx == kNone || v[i] > best)) {
          best = v[i];
          bidx = j;
        }
      }
    };
    double lb;
    int li;
    local_best(lb, li);
    for (int round = 0; round < kb; ++round) {
      double best = lb;
      int bidx = li;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const double ob = __shfl_xor_sync(0xffffffffu, best, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bidx, off);
        if (oi != kNone && (bidx == kNone || ob > best || (ob == best && oi < bidx))) {
          best = ob;
          bidx = oi;
        }
      }
      if (bidx != kNone && (bidx & 31) == lane) {
        taken |= 1u << (bidx >> 5);
        local_best(lb, li);
      }
    }
  }
  int pos = 0;
#pragma unroll
  for (int i = 0; i < MAXP; ++i) {
    const int j = i * 32 + lane;
    const bool mine = j < nb && ((taken >> i) & 1u);
    const uint32_t ball = __ballot_sync(0xffffffffu, mine);
    if (mine) out[pos + __popc(ball & ((1u << lane) - 1u))] = j;
    pos += __popc(ball);
  }
}

template <int MAXP>
static void launch_topk(const double* sigma, int32_t* idx, int rows, int nb, int kb, const int32_t* kb_h,
                        int H, int32_t* dev_err, cudaStream_t cs) {
  topk_kernel<MAXP><<<(rows + kTopkWarps - 1) / kTopkWarps, kTopkWarps * 32, 0, cs>>>(
      sigma, idx, rows, nb, kb, kb_h, H, dev_err);
}

// Scores and top-k from pooled block means (float64 [B, H, nb, d]); kb_h:
// optional per-head kept counts (device int32 [H]).
rola_status_t select_from_pooled(const rola_shape_t* s, const double* qbar, const double* kbar,
                                 double* sigma, int32_t* idx, cudaStream_t cs, const int32_t* kb_h,
                                 int32_t* dev_err) {
  const int nb = rola_num_blocks(s);
  const int tiles = (nb + kScTile - 1) / kScTile;
  if (cudaFuncSetAttribute(score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kScSmemBytes) !=
      cudaSuccess)
    return ROLA_ERR_CUDA;
  score_kernel<<<dim3(tiles, tiles, s->B * s->H), 128, kScSmemBytes, cs>>>(qbar, kbar, sigma, s->H, s->d, nb);
  const int rows = s->B * s->H * nb;
  const int nper = (nb + 31) / 32;
  const int H = s->H, kb = s->k_b;
  if (nper <= 4) launch_topk<4>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  else if (nper <= 8) launch_topk<8>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  else if (nper <= 16) launch_topk<16>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  else if (nper <= 20) launch_topk<20>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  else if (nper <= 24) launch_topk<24>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  else launch_topk<kMaxPerLane>(sigma, idx, rows, nb, kb, kb_h, H, dev_err, cs);
  return cudaGetLastError() == cudaSuccess ? ROLA_OK : ROLA_ERR_CUDA;
}

}  // namespace rola

using namespace rola;

extern "C" size_t rola_select_workspace_bytes(const rola_shape_t* s) {
  if (rola_internal::check_shape(s) != ROLA_OK) return 0;
  const size_t nb = (size_t)rola_num_blocks(s);
  const size_t pooled = 2 * (size_t)s->B * s->H * nb * s->d * sizeof(double);
  const size_t scores = (size_t)s->B * s->H * nb * nb * sizeof(double);
  return rola_internal::round_up(pooled, 256) + rola_internal::round_up(scores, 256);
}

extern "C" size_t rola_workspace_bytes(const rola_shape_t* s) { return rola_select_workspace_bytes(s); }

extern "C" rola_status_t rola_select_blocks(const rola_shape_t* s, const uint16_t* q,
                                            const uint16_t* k, int32_t* idx, double* scores_opt,
                                            void* ws, size_t ws_bytes, void* stream) {
  return select_blocks_impl(s, nullptr, q, k, idx, scores_opt, ws, ws_bytes, nullptr, stream);
}

rola_status_t rola::select_blocks_impl(const rola_shape_t* s, const int32_t* kb_h, const uint16_t* q,
                                       const uint16_t* k, int32_t* idx, double* scores_opt, void* ws,
                                       size_t ws_bytes, int32_t* dev_err, void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q || !k || !idx) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(q, 16) || !rola_host::aligned(k, 16) || !rola_host::aligned(idx, 4) ||
      (scores_opt && !rola_host::aligned(scores_opt, 8)))
    return ROLA_ERR_ALIGNMENT;
  const int nb = rola_num_blocks(s);
  if (nb > 32 * kMaxPerLane) return ROLA_ERR_UNSUPPORTED;
  const size_t need = rola_select_workspace_bytes(s);
  if (!ws || ws_bytes < need || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  double* qbar = reinterpret_cast<double*>(ws);
  double* kbar = qbar + (size_t)s->B * s->H * nb * s->d;
  double* sig = reinterpret_cast<double*>(
      reinterpret_cast<char*>(ws) +
      rola_internal::round_up(2 * (size_t)s->B * s->H * nb * s->d * sizeof(double), 256));
  if (scores_opt) sig = scores_opt;

  pool_kernel<<<dim3(nb, s->B, 2), 256, 0, cs>>>(q, k, qbar, kbar, s->N, s->H, s->d, s->block, nb);
  if (cudaGetLastError() != cudaSuccess) return ROLA_ERR_CUDA;
  return select_from_pooled(s, qbar, kbar, sig, idx, cs, kb_h, dev_err);
}

// ---------------------------------------------------------------- selector without a workspace
// The same selector (pooling, scores, top-k: the kernels above) with its
// scratch in a fixed device array of this library instead of a caller
// workspace.  It serves callers that cannot hand over device memory at the
// call site: a host-side plugin or language binding that holds only the q, k
// and idx buffers and has no device allocator of its own.  Nothing is
// allocated per call: the array exists once per device for the life of the
// context.  In host code the array's name is only a stand-in, so every call
// asks the runtime for its device address on the current device
// (cudaGetSymbolAddress).  That lookup is cheap once the library's module is
// loaded on the device; the first call on a device loads it, so that first
// call should come before any stream capture.  Asking on every call (instead
// of caching the address) keeps the entry point correct after a device reset
// or a re-created primary context, where the array has a new address.  Every
// scratch word is written before it is read, so nothing needs clearing
// between calls; calls that overlap in time on one device (several streams or
// host threads) share the array and race.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

namespace {

// Device address of the scratch array on the current device, or null.
void* scratch_on_current_device() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess) return nullptr;
  return p;
}

}  // namespace

extern "C" rola_status_t rola_select_blocks_noalloc(const rola_shape_t* s, const uint16_t* q,
                                                    const uint16_t* k, int32_t* idx, void* stream) {
  rola_status_t st = rola_internal::check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q || !k || !idx) return ROLA_ERR_INVALID_ARG;
  if (!rola_host::aligned(q, 16) || !rola_host::aligned(k, 16) || !rola_host::aligned(idx, 4))
    return ROLA_ERR_ALIGNMENT;
  const int nb = rola_num_blocks(s);
  if (nb > 32 * kMaxPerLane) return ROLA_ERR_UNSUPPORTED;
  // the scratch this shape needs must fit the fixed array
  if (rola_select_workspace_bytes(s) > kNoAllocScratchBytes) return ROLA_ERR_WORKSPACE;
  char* ws = static_cast<char*>(scratch_on_current_device());
  if (!ws) return ROLA_ERR_CUDA;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  double* qbar = reinterpret_cast<double*>(ws);
  double* kbar = qbar + (size_t)s->B * s->H * nb * s->d;
  double* sig = reinterpret_cast<double*>(
      ws + rola_internal::round_up(2 * (size_t)s->B * s->H * nb * s->d * sizeof(double), 256));
  pool_kernel<<<dim3(nb, s->B, 2), 256, 0, cs>>>(q, k, qbar, kbar, s->N, s->H, s->d, s->block, nb);
  if (cudaGetLastError() != cudaSuccess) return ROLA_ERR_CUDA;
  return select_from_pooled(s, qbar, kbar, sig, idx, cs, nullptr, nullptr);
}
