// Host side of the librola C ABI: status strings, shape validation, the
// kept-block rule, rotary frequency table, driver entry point for tensor-map
// encoding, and the whole-layer entry points that chain the kernels.
#include <math.h>
#include <string.h>

#include <mutex>

#include "rola_common.cuh"
#include "rola_internal.h"

namespace rola_internal {

rola_status_t check_shape(const rola_shape_t* s) {
  if (!s) return ROLA_ERR_INVALID_ARG;
  if (s->B < 1 || s->H < 1 || s->T < 1 || s->Hg < 1 || s->W < 1 || s->d < 1 || s->r < 1 ||
      s->block < 1)
    return ROLA_ERR_INVALID_ARG;
  const long long N = (long long)s->T * s->Hg * s->W;
  if (N != s->N || N > (1LL << 30)) return ROLA_ERR_INVALID_ARG;
  if ((long long)s->B * N * s->H * s->d >= (1LL << 40)) return ROLA_ERR_INVALID_ARG;
  const int nb = (int)((N + s->block - 1) / s->block);
  if (s->k_b < 1 || s->k_b > nb) return ROLA_ERR_INVALID_ARG;
  if (s->r % 2 != 0 || s->r > s->d) return ROLA_ERR_INVALID_ARG;
  if (!(s->rope_base > 0.f) || !isfinite(s->rope_base)) return ROLA_ERR_INVALID_ARG;
  if (s->d != 64 && s->d != 128) return ROLA_ERR_UNSUPPORTED;
  if (s->block != 64 && s->block != 128) return ROLA_ERR_UNSUPPORTED;
  if (s->r != 16 && s->r != 32) return ROLA_ERR_UNSUPPORTED;
  return ROLA_OK;
}

LayerWs layer_ws(const rola_shape_t* s) {
  LayerWs w{};
  const size_t nb = (size_t)rola_num_blocks(s);
  const size_t BH = (size_t)s->B * s->H;
  size_t off = 0;
  w.select = off;
  off += round_up(rola_select_workspace_bytes(s), 256);
  w.idx = off;
  off += round_up(BH * nb * s->k_b * sizeof(int32_t), 256);
  w.S_blk = off;
  off += round_up(BH * nb * s->r * s->d * sizeof(float), 256);
  w.z_blk = off;
  off += round_up(BH * nb * s->r * sizeof(float), 256);
  w.S_glb = off;
  off += round_up(BH * s->r * s->d * sizeof(float), 256);
  w.z_glb = off;
  off += round_up(BH * s->r * sizeof(float), 256);
  w.total = off;
  return w;
}

}  // namespace rola_internal

namespace rola_host {

EncodeTiledFn encode_tiled_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int rope_frequencies(int r, float base, double* freq, int* axis) {
  const int rh = 2 * (r / 6);
  const int split[3] = {r - 2 * rh, rh, rh};
  int p = 0;
  for (int ax = 0; ax < 3; ++ax)
    for (int m = 0; m < split[ax] / 2; ++m) {
      freq[p] = pow((double)base, -2.0 * m / split[ax]);
      axis[p] = ax;
      ++p;
    }
  return p;
}

void rope_table_layout(const rola_shape_t* s, const int* axis, RopeTabLayout* out) {
  const int npairs = s->r / 2;
  const int len[3] = {s->T, s->Hg, s->W};
  int np_axis[3] = {0, 0, 0};
  for (int pr = 0; pr < npairs; ++pr) ++np_axis[axis[pr]];
  const long long off[3] = {0, (long long)len[0] * np_axis[0],
                            (long long)len[0] * np_axis[0] + (long long)len[1] * np_axis[1]};
  int first = 0, m_axis[3] = {0, 0, 0};
  for (int pr = 0; pr < npairs; ++pr) {
    const int ax = axis[pr];
    out->base[pr] = (int)(off[ax] + m_axis[ax]++);
    out->stride[pr] = np_axis[ax];
    out->first[pr] = first;
    first += len[ax];
  }
  out->first[npairs] = first;
  out->entries = (int)(off[2] + (long long)len[2] * np_axis[2]);
}

bool make_act_map(CUtensorMap* m, const void* base, const rola_shape_t* s, int box_rows) {
  auto enc = encode_tiled_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {(cuuint64_t)s->d, (cuuint64_t)s->H, (cuuint64_t)s->N, (cuuint64_t)s->B};
  const cuuint64_t strides[3] = {(cuuint64_t)s->d * 2, (cuuint64_t)s->H * s->d * 2,
                                 (cuuint64_t)s->N * s->H * s->d * 2};
  const cuuint32_t box[4] = {64, 1, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

}  // namespace rola_host

using rola_internal::check_shape;
using rola_internal::round_up;

extern "C" const char* rola_status_string(rola_status_t s) {
  switch (s) {
    case ROLA_OK: return "ok";
    case ROLA_ERR_INVALID_ARG: return "invalid argument";
    case ROLA_ERR_UNSUPPORTED: return "unsupported shape";
    case ROLA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    case ROLA_ERR_CUDA: return "CUDA error";
    case ROLA_ERR_ALIGNMENT: return "pointer misaligned";
  }
  return "unknown status";
}

extern "C" int32_t rola_num_blocks(const rola_shape_t* s) {
  if (!s || s->block < 1 || s->N < 1) return -1;
  return (int32_t)(((long long)s->N + s->block - 1) / s->block);
}

extern "C" int32_t rola_kb_from_sparsity(int32_t n_blocks, int32_t sparsity_permille) {
  if (n_blocks < 1 || sparsity_permille < 0 || sparsity_permille >= 1000) return -1;
  const long long keep = (long long)(1000 - sparsity_permille) * n_blocks;
  return (int32_t)((keep + 999) / 1000);
}

extern "C" size_t rola_layer_workspace_bytes(const rola_shape_t* s) {
  if (check_shape(s) != ROLA_OK) return 0;
  return rola_internal::layer_ws(s).total;
}

extern "C" int rola_layer_kernel_launches(const rola_shape_t* s) {
  if (check_shape(s) != ROLA_OK) return 0;
  // fused path: prep, score, top-k, state totals, attention;
  // otherwise: pool, score, top-k, block states, state totals, attention
  return rola::prep_kernel_supports(s) ? 5 : 6;
}

extern "C" rola_status_t rola_layer_fwd(const rola_shape_t* s, const uint16_t* q, const uint16_t* k,
                                        const uint16_t* v, const uint16_t* P, const float* gate,
                                        uint16_t* out, int32_t* idx_out, void* ws, size_t ws_bytes,
                                        int32_t* dev_err, void* stream) {
  return rola_layer_fwd_timed(s, q, k, v, P, gate, out, idx_out, ws, ws_bytes, dev_err, stream, nullptr, 0);
}

namespace {
// The layer: selection (or a given mask), block states, attention.  kb_h:
// optional per-head kept counts (device int32 [H]); reuse: idx_io is the mask
// to use and no selection runs; otherwise the selected mask is copied to
// idx_io when it is not NULL.
rola_status_t layer_run(const rola_shape_t* s, const int32_t* kb_h, bool reuse, const uint16_t* q,
                        const uint16_t* k, const uint16_t* v, const uint16_t* P, const float* gate,
                        uint16_t* out, int32_t* idx_io, void* ws, size_t ws_bytes, int32_t* dev_err,
                        void* stream, void* const* events, int32_t n_events) {
  if (events && n_events != 3 && n_events != 5) return ROLA_ERR_INVALID_ARG;
  if (reuse && (!idx_io || !rola_host::aligned(idx_io, 4))) return idx_io ? ROLA_ERR_ALIGNMENT : ROLA_ERR_INVALID_ARG;
  // stage boundaries 0..4 (start, after the q/k/v pass, after scores and
  // top-k, after the totals, end); three events keep stages 0, 3 and 4
  auto mark = [&](int stage) -> bool {
    if (!events) return true;
    const int i = n_events == 5 ? stage : (stage == 0 ? 0 : stage == 3 ? 1 : stage == 4 ? 2 : -1);
    return i < 0 || cudaEventRecord(reinterpret_cast<cudaEvent_t>(events[i]),
                                    reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess;
  };
  rola_status_t st = check_shape(s);
  if (st != ROLA_OK) return st;
  const rola_internal::LayerWs L = rola_internal::layer_ws(s);
  if (!ws || ws_bytes < L.total || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  char* base = reinterpret_cast<char*>(ws);
  int32_t* idx = reuse ? idx_io : reinterpret_cast<int32_t*>(base + L.idx);
  float* S_blk = reinterpret_cast<float*>(base + L.S_blk);
  float* z_blk = reinterpret_cast<float*>(base + L.z_blk);
  float* S_glb = reinterpret_cast<float*>(base + L.S_glb);
  float* z_glb = reinterpret_cast<float*>(base + L.z_glb);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (!mark(0)) return ROLA_ERR_CUDA;
  if (rola::prep_kernel_supports(s)) {
    // one pass over q, k, v: block means for the selector and block states
    if (!q || !k || !v || !P || !gate || !out) return ROLA_ERR_INVALID_ARG;
    if (!rola_host::aligned(q, 16) || !rola_host::aligned(k, 16) || !rola_host::aligned(v, 16) ||
        !rola_host::aligned(P, 16))
      return ROLA_ERR_ALIGNMENT;
    if (rola_num_blocks(s) > 1024) return ROLA_ERR_UNSUPPORTED;
    const size_t pooled = (size_t)s->B * s->H * rola_num_blocks(s) * s->d;
    double* qbar = reinterpret_cast<double*>(base + L.select);
    double* kbar = qbar + pooled;
    double* sigma = reinterpret_cast<double*>(base + L.select + round_up(2 * pooled * sizeof(double), 256));
    st = rola::launch_prep_kernel(s, q, k, v, P, qbar, kbar, S_blk, z_blk, dev_err, cs);
    if (st != ROLA_OK) return st;
    if (!mark(1)) return ROLA_ERR_CUDA;
    if (!reuse) {
      st = rola::select_from_pooled(s, qbar, kbar, sigma, idx, cs, kb_h, dev_err);
      if (st != ROLA_OK) return st;
    }
    if (!mark(2)) return ROLA_ERR_CUDA;
    st = rola::launch_states_total(s, S_blk, z_blk, S_glb, z_glb, cs);
    if (st != ROLA_OK) return st;
  } else {
    if (!reuse) {
      st = rola::select_blocks_impl(s, kb_h, q, k, idx, nullptr, base + L.select, L.idx - L.select, dev_err,
                                    stream);
      if (st != ROLA_OK) return st;
    }
    if (!mark(1) || !mark(2)) return ROLA_ERR_CUDA;
    st = rola_block_states(s, k, v, P, S_blk, z_blk, S_glb, z_glb, stream);
    if (st != ROLA_OK) return st;
  }
  if (!mark(3)) return ROLA_ERR_CUDA;
  st = rola::attention_launch(s, kb_h, q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate, out, dev_err,
                              rola::kWaitLimitNs, stream);
  if (st != ROLA_OK) return st;
  if (!mark(4)) return ROLA_ERR_CUDA;
  if (idx_io && !reuse) {
    const size_t bytes = (size_t)s->B * s->H * rola_num_blocks(s) * s->k_b * sizeof(int32_t);
    if (cudaMemcpyAsync(idx_io, idx, bytes, cudaMemcpyDeviceToDevice,
                        reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
      return ROLA_ERR_CUDA;
  }
  return ROLA_OK;
}
}  // namespace

extern "C" rola_status_t rola_layer_fwd_timed(const rola_shape_t* s, const uint16_t* q,
                                              const uint16_t* k, const uint16_t* v, const uint16_t* P,
                                              const float* gate, uint16_t* out, int32_t* idx_out,
                                              void* ws, size_t ws_bytes, int32_t* dev_err, void* stream,
                                              void* const* events, int32_t n_events) {
  return layer_run(s, nullptr, false, q, k, v, P, gate, out, idx_out, ws, ws_bytes, dev_err, stream, events,
                   n_events);
}

extern "C" rola_status_t rola_layer_fwd_ex(const rola_shape_t* s, const rola_layer_opts_t* opts,
                                           const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                           const uint16_t* P, const float* gate, uint16_t* out,
                                           int32_t* idx_io, void* ws, size_t ws_bytes, int32_t* dev_err,
                                           void* stream, void* const* events, int32_t n_events) {
  const int32_t* kb_h = opts ? opts->kb_per_head : nullptr;
  if (kb_h && !rola_host::aligned(kb_h, 4)) return ROLA_ERR_ALIGNMENT;
  return layer_run(s, kb_h, opts && opts->reuse_mask, q, k, v, P, gate, out, idx_io, ws, ws_bytes, dev_err,
                   stream, events, n_events);
}

namespace {
// The host-buffer layer runs in head groups: (batch, head) pairs are
// independent, so while one group computes, the next group's q, k, v cross
// PCIe and the previous group's output goes back.  A group holds heads whose
// slice of a token row is at least 2 KB (8 heads of d = 128), so that the
// strided copies move long rows.
constexpr int kHostGroupRowBytes = 2048;

int host_group_heads(const rola_shape_t* s) {
  const int row = s->d * (int)sizeof(uint16_t);
  const int hc = (kHostGroupRowBytes + row - 1) / row;
  return hc < s->H ? hc : s->H;
}

rola_shape_t group_shape(const rola_shape_t* s, int heads) {
  rola_shape_t g = *s;
  g.H = heads;
  return g;
}

// Device staging: P and gate of all heads, two slots of (q, k, v, out) of
// one group, compact [B, N, hc, d], and the layer workspace of one group.
struct HostWs {
  size_t P, gate, slot[2], q, k, v, out, slot_bytes, layer, total;
};
HostWs host_ws(const rola_shape_t* s) {
  using rola_internal::round_up;
  HostWs w{};
  const rola_shape_t g = group_shape(s, host_group_heads(s));
  const size_t act = round_up((size_t)g.B * g.N * g.H * g.d * sizeof(uint16_t), 256);
  size_t off = 0;
  w.P = off; off += round_up((size_t)s->H * s->d * s->r * sizeof(uint16_t), 256);
  w.gate = off; off += round_up((size_t)s->H * sizeof(float), 256);
  w.q = 0; w.k = act; w.v = 2 * act; w.out = 3 * act;
  w.slot_bytes = 4 * act;
  w.slot[0] = off; off += w.slot_bytes;
  w.slot[1] = off; off += w.slot_bytes;
  w.layer = off; off += rola_internal::layer_ws(&g).total;
  w.total = off;
  return w;
}

// Copy streams and the events that order them against the caller's stream,
// created once per device and kept for the life of the process.  Enqueueing
// a call holds the device's lock, so concurrent calls cannot interleave their
// event records.
struct HostPipe {
  bool ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in[2] = {}, done[2] = {}, out[2] = {};
  std::mutex lock;
};
constexpr int kMaxDevices = 64;
HostPipe g_pipes[kMaxDevices];
std::mutex g_pipes_lock;

HostPipe* host_pipe() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> guard(g_pipes_lock);
  HostPipe& hp = g_pipes[dev];
  if (!hp.ready) {
    bool ok = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < 2; ++i)
      ok = cudaEventCreateWithFlags(&hp.in[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.done[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.out[i], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) return nullptr;
    hp.ready = true;
  }
  return &hp;
}
}  // namespace

extern "C" size_t rola_layer_host_workspace_bytes(const rola_shape_t* s) {
  if (check_shape(s) != ROLA_OK) return 0;
  return host_ws(s).total;
}

extern "C" rola_status_t rola_layer_fwd_host(const rola_shape_t* s, const uint16_t* q_host,
                                             const uint16_t* k_host, const uint16_t* v_host,
                                             const uint16_t* P_host, const float* gate_host,
                                             uint16_t* out_host, void* ws, size_t ws_bytes,
                                             int32_t* dev_err, void* stream) {
  const rola_status_t st = check_shape(s);
  if (st != ROLA_OK) return st;
  if (!q_host || !k_host || !v_host || !P_host || !gate_host || !out_host)
    return ROLA_ERR_INVALID_ARG;
  const HostWs w = host_ws(s);
  if (!ws || ws_bytes < w.total || !rola_host::aligned(ws, 256)) return ROLA_ERR_WORKSPACE;
  HostPipe* hp = host_pipe();
  if (!hp) return ROLA_ERR_CUDA;
  std::lock_guard<std::mutex> guard(hp->lock);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(ws);
  const int hc = host_group_heads(s);
  const int groups = (s->H + hc - 1) / hc;
  const size_t rows = (size_t)s->B * s->N;
  const size_t row_bytes = (size_t)s->H * s->d * sizeof(uint16_t);  // one token of all heads
  const size_t head_bytes = (size_t)s->d * sizeof(uint16_t);
  const size_t pbytes = (size_t)s->H * s->d * s->r * sizeof(uint16_t);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };
  // everything before this call on `stream` (e.g. the last use of ws) first
  if (!ok(cudaEventRecord(hp->start, cs)) || !ok(cudaStreamWaitEvent(hp->h2d, hp->start, 0)) ||
      !ok(cudaStreamWaitEvent(hp->d2h, hp->start, 0)))
    return ROLA_ERR_CUDA;
  rola_status_t result = ROLA_OK;
  if (!ok(cudaMemcpyAsync(base + w.P, P_host, pbytes, cudaMemcpyHostToDevice, hp->h2d)) ||
      !ok(cudaMemcpyAsync(base + w.gate, gate_host, (size_t)s->H * sizeof(float),
                          cudaMemcpyHostToDevice, hp->h2d)))
    result = ROLA_ERR_CUDA;
  for (int gi = 0; result == ROLA_OK && gi < groups; ++gi) {
    const int sl = gi & 1;
    const int h0 = gi * hc;
    const int heads = s->H - h0 < hc ? s->H - h0 : hc;
    const size_t width = (size_t)heads * head_bytes;  // this group's slice of a token row
    char* slot = base + w.slot[sl];
    // inputs: the slot's previous group must have finished computing
    if (gi >= 2 && !ok(cudaStreamWaitEvent(hp->h2d, hp->done[sl], 0))) {
      result = ROLA_ERR_CUDA;
      break;
    }
    const uint16_t* src[3] = {q_host, k_host, v_host};
    const size_t dst_off[3] = {w.q, w.k, w.v};
    bool copied = true;
    for (int t = 0; copied && t < 3; ++t)
      copied = ok(cudaMemcpy2DAsync(slot + dst_off[t], width,
                                    reinterpret_cast<const char*>(src[t]) + (size_t)h0 * head_bytes,
                                    row_bytes, width, rows, cudaMemcpyHostToDevice, hp->h2d));
    if (!copied || !ok(cudaEventRecord(hp->in[sl], hp->h2d))) {
      result = ROLA_ERR_CUDA;
      break;
    }
    // compute on the caller's stream once the inputs are in and the slot's
    // previous output has gone back
    if (!ok(cudaStreamWaitEvent(cs, hp->in[sl], 0)) ||
        (gi >= 2 && !ok(cudaStreamWaitEvent(cs, hp->out[sl], 0)))) {
      result = ROLA_ERR_CUDA;
      break;
    }
    const rola_shape_t g = group_shape(s, heads);
    result = rola_layer_fwd(&g, reinterpret_cast<uint16_t*>(slot + w.q),
                            reinterpret_cast<uint16_t*>(slot + w.k),
                            reinterpret_cast<uint16_t*>(slot + w.v),
                            reinterpret_cast<uint16_t*>(base + w.P) + (size_t)h0 * s->d * s->r,
                            reinterpret_cast<float*>(base + w.gate) + h0,
                            reinterpret_cast<uint16_t*>(slot + w.out), nullptr, base + w.layer,
                            w.total - w.layer, dev_err, stream);
    if (result != ROLA_OK) break;
    if (!ok(cudaEventRecord(hp->done[sl], cs))) {
      result = ROLA_ERR_CUDA;
      break;
    }
    // output of this group back into its columns of the host rows
    if (!ok(cudaStreamWaitEvent(hp->d2h, hp->done[sl], 0)) ||
        !ok(cudaMemcpy2DAsync(reinterpret_cast<char*>(out_host) + (size_t)h0 * head_bytes,
                              row_bytes, slot + w.out, width, width, rows, cudaMemcpyDeviceToHost,
                              hp->d2h)) ||
        !ok(cudaEventRecord(hp->out[sl], hp->d2h))) {
      result = ROLA_ERR_CUDA;
      break;
    }
  }
  // whatever happened above, the caller's stream continues only after every
  // copy this call enqueued (on success the last ones are the copies back)
  const bool joined = ok(cudaEventRecord(hp->in[0], hp->h2d)) &&
                      ok(cudaStreamWaitEvent(cs, hp->in[0], 0)) &&
                      ok(cudaEventRecord(hp->out[0], hp->d2h)) &&
                      ok(cudaStreamWaitEvent(cs, hp->out[0], 0));
  return result != ROLA_OK ? result : (joined ? ROLA_OK : ROLA_ERR_CUDA);
}
