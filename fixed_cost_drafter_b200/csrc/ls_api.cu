// Host side of the C ABI declared in include/longspark.h: argument validation, the
// state arena layout, and the kernel launches. No entry point allocates device memory.
#include <cstdlib>
#include <cstring>
#include <new>

#include "ls_common.cuh"
#include "ls_attend_tc.h"

namespace ls {
cudaError_t launch_commit(const Dev& p, const int32_t* draft, const int32_t* target, const void* vk,
                          const void* vv, const void* vh, int32_t* accept_len, int32_t* next_token,
                          const int32_t* given_a, cudaStream_t stream);
bool prologue_supported(const Dev& p);
cudaError_t launch_prologue(const Dev& p, const void* w_kv, const void* w_q, const void* x, void* bkv, void* q,
                            int sms, cudaStream_t stream);
cudaError_t launch_sample(const Dev& p, const int32_t* draft, const float* q, const float* pr, int vocab,
                          const float* u, int32_t* accept_len, int32_t* next_token, cudaStream_t stream);
bool simt_supported(const Dev& p);
cudaError_t launch_attend_simt(const Dev& p, int lb, int lcount, const void* q, const void* bk,
                               const void* bv, int64_t bstride, float scale, int views, void* out,
                               cudaStream_t stream);
size_t prefill_workspace_bytes(const ls_config& c, int64_t row_begin, int64_t row_end);
cudaError_t launch_prefill(const Dev& p, const ls_config& c, const void* k, const void* v,
                           int64_t plane_stride, int64_t row_stride, const int64_t* prefix_len,
                           int64_t row_begin, int64_t row_end, const void* last_hidden, void* ws,
                           int sms, cudaStream_t stream);
cudaError_t launch_commit_paged(const Dev& p, const int32_t* draft, const int32_t* target, const ls_paged_kv& kv,
                                const void* vh, int32_t* accept_len, int32_t* next_token, const int32_t* given_a,
                                cudaStream_t stream);
cudaError_t launch_prefill_paged(const Dev& p, const ls_config& c, const ls_paged_kv& kv, const int64_t* prefix_len,
                                 int64_t row_begin, int64_t row_end, const void* last_hidden, void* ws, int sms,
                                 cudaStream_t stream);
size_t noalloc_scratch_bytes();
cudaError_t noalloc_scratch(int device, void** out);
cudaError_t launch_wait_timeout(const Dev& p, uint32_t polls, cudaStream_t stream);
}  // namespace ls

struct ls_state {
  ls_config cfg;
  ls::Layout lay;
  ls::Dev dev;
  void* arena;
  int device;
  int sms;
  int use_tc;
  ls::TcPlan tc;
  // No call has written the views since a launch on settled_stream after which every
  // earlier writer has completed before the next kernel on that stream starts (see
  // mark_settled): an attention launched next on that stream may load its first K/V chunks
  // before its grid dependency wait (ls::kAttendViewsSettled).
  // (kept by the calls that only read the state too: mutable)
  mutable int views_settled;
  mutable cudaStream_t settled_stream;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// A state belongs to the device that was current at ls_init_state: its arena, tensor maps
// and the library's fixed scratch are that device's. Calls made while another device is
// current are refused.
bool on_state_device(const ls_state* st) {
  int dev = -1;
  return cudaGetDevice(&dev) == cudaSuccess && dev == st->device;
}

// After a launch on `stream` that writes no views and lets the kernels behind it start only
// once everything before it has completed (it triggers its dependents after its grid
// dependency wait, or it is launched without programmatic serialization), every call that
// wrote the views has completed by the time a kernel launched next on `stream` starts.
// A launch captured into a graph runs only when the graph is launched, in an order the host
// does not see: it settles nothing for the launches made on the stream after the capture
// (which follow whatever was launched before it), so the state is left unsettled.
void mark_settled(const ls_state* st, cudaStream_t stream) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  const bool captured = cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone;
  st->views_settled = captured ? 0 : 1;
  st->settled_stream = stream;
}
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int validate(const ls_config* c) {
  if (!c) return LS_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_layers < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 ||
      c->head_dim < 1 || c->hidden < 1 || c->block < 1 || c->window < 1 || c->n_scales < 1 ||
      c->slots_per_scale < 1)
    return LS_ERR_INVALID_ARG;
  if (c->dtype != LS_F32 && c->dtype != LS_BF16) return LS_ERR_INVALID_ARG;
  if (c->n_scales > LS_MAX_SCALES) return LS_ERR_UNSUPPORTED;
  if (c->n_q_heads % c->n_kv_heads != 0) return LS_ERR_SHAPE;
  if (c->window < c->block + 1) return LS_ERR_SHAPE;  // a round's rows get distinct slots
  for (int k = 0; k < c->n_scales; ++k) {
    if (c->scales[k] < 1) return LS_ERR_INVALID_ARG;
    if (k > 0 && c->scales[k] <= c->scales[k - 1]) return LS_ERR_SHAPE;
  }
  // GPU-path limits (valid for the method, not handled by these kernels)
  if (c->scales[0] < c->block + 1) return LS_ERR_UNSUPPORTED;  // <= 1 close per scale per round
  for (int k = 1; k < c->n_scales; ++k)
    if (c->scales[k] % c->scales[k - 1] != 0) return LS_ERR_UNSUPPORTED;
  const int elem = c->dtype == LS_BF16 ? 2 : 4;
  if (c->head_dim % 8 != 0 || c->head_dim > 256 || c->hidden % 8 != 0) return LS_ERR_UNSUPPORTED;
  const int lanes = c->head_dim * elem / 16;
  if (!pow2(lanes) || lanes > 32) return LS_ERR_UNSUPPORTED;
  if (c->n_kv_heads > 8 || c->block > 32) return LS_ERR_UNSUPPORTED;
  if (c->flags & ~(LS_FLAG_FORCE_SIMT | LS_FLAG_OUT_F32)) return LS_ERR_INVALID_ARG;
  return LS_OK;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LS_OK : LS_ERR_CUDA; }

// A paged-cache descriptor usable by the kernels for this config: every tapped layer's
// pages given and 16-byte aligned, packed rows of all KV heads, strides in whole
// 16-byte steps (8 elements), a block table and at least one page.
int validate_paged(const ls_config& c, const ls_paged_kv* kv) {
  if (!kv) return LS_ERR_INVALID_ARG;
  if (c.n_layers > LS_MAX_PAGED_LAYERS) return LS_ERR_UNSUPPORTED;
  for (int l = 0; l < c.n_layers; ++l) {
    if (!kv->k_layers[l] || !kv->v_layers[l]) return LS_ERR_INVALID_ARG;
    if (!aligned16(kv->k_layers[l]) || !aligned16(kv->v_layers[l])) return LS_ERR_INVALID_ARG;
  }
  if (!kv->block_table || kv->page_size < 1 || kv->max_blocks < 1 || kv->num_pages < 1) return LS_ERR_INVALID_ARG;
  if (kv->verify_slots && (reinterpret_cast<uintptr_t>(kv->verify_slots) & 7) != 0) return LS_ERR_INVALID_ARG;
  if (kv->slot_stride < int64_t(c.n_kv_heads) * c.head_dim || kv->slot_stride % 8 != 0 ||
      kv->page_stride < 0 || kv->page_stride % 8 != 0)
    return LS_ERR_SHAPE;
  return LS_OK;
}

// Argument checks of the whole-round calls beyond those of the commit they make.
int round_checks(const ls_state* st, int64_t boundary_k_offset, int64_t boundary_v_offset, float softmax_scale,
                 const void* d_q, const void* d_out) {
  const ls_config& c = st->cfg;
  const int64_t span = int64_t(c.n_kv_heads) * c.head_dim;
  if (boundary_k_offset < 0 || boundary_v_offset < 0 || boundary_k_offset % 8 != 0 ||
      boundary_v_offset % 8 != 0 || boundary_k_offset + span > c.hidden || boundary_v_offset + span > c.hidden)
    return LS_ERR_SHAPE;
  if (!(softmax_scale > 0.0f) || softmax_scale == INFINITY) return LS_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_out)) return LS_ERR_INVALID_ARG;
  return LS_OK;
}

// The attention half of a whole round (after its commit was enqueued).
int round_attend(ls_state* st, const void* d_q, int64_t boundary_k_offset, int64_t boundary_v_offset,
                 float softmax_scale, void* d_out, cudaStream_t stream);

}  // namespace

extern "C" {

const char* ls_status_string(int s) {
  switch (s) {
    case LS_OK: return "ok";
    case LS_ERR_INVALID_ARG: return "invalid argument";
    case LS_ERR_SHAPE: return "inconsistent shapes";
    case LS_ERR_UNSUPPORTED: return "unsupported by the GPU path";
    case LS_ERR_CUDA: return "CUDA runtime error";
    case LS_ERR_DEVICE: return "device error word set";
    case LS_ERR_DEVICE_TIMEOUT: return "bounded device wait timed out";
    case LS_ERR_SCRATCH_LIMIT: return "needs more than the library's fixed 16 MiB scratch: split the prefix into chunks";
    default: return "unknown status";
  }
}

size_t ls_state_bytes(const ls_config* cfg) {
  if (validate(cfg) != LS_OK) return 0;
  return size_t(ls::make_layout(*cfg).total);
}

size_t ls_view_state_bytes(const ls_config* cfg, int32_t views) {
  if (validate(cfg) != LS_OK || (views & ~LS_VIEW_ALL)) return 0;
  const ls_config& c = *cfg;
  const int64_t e = c.dtype == LS_BF16 ? 2 : 4;
  const int64_t bl = int64_t(c.batch) * c.n_layers, tiles = bl * c.n_kv_heads;
  const int64_t summary_rows = int64_t(c.n_scales) * (c.slots_per_scale + 1) + 1;
  int64_t n = bl * (1 + c.n_scales) * 8;  // counters
  if (views & LS_VIEW_WINDOW) n += tiles * 2 * c.window * c.head_dim * e;
  if (views & LS_VIEW_SUMMARY) n += tiles * 2 * summary_rows * c.head_dim * (4 + e);
  if (views & LS_VIEW_BOUNDARY) n += bl * c.hidden * e;
  return size_t(n);
}

int ls_get_layout(const ls_config* cfg, ls_layout* out) {
  const int v = validate(cfg);
  if (v != LS_OK) return v;
  if (!out) return LS_ERR_INVALID_ARG;
  const ls::Layout y = ls::make_layout(*cfg);
  out->total_bytes = size_t(y.total);
  out->off_counters = size_t(y.counters);
  out->off_error = size_t(y.error);
  out->off_sync = size_t(y.sync);
  out->off_kv = size_t(y.kv);
  out->off_seg_mean = size_t(y.seg);
  out->off_part_sum = size_t(y.part);
  out->off_glob_sum = size_t(y.glob);
  out->off_boundary = size_t(y.boundary);
  out->off_sample = size_t(y.sample);
  out->off_prologue = size_t(y.prologue);
  out->kv_rows = y.R;
  out->elem_bytes = y.elem;
  return LS_OK;
}

int ls_init_state(const ls_config* cfg, void* d_arena, size_t arena_bytes, ls_state** out,
                  cudaStream_t stream) {
  const int v = validate(cfg);
  if (v != LS_OK) return v;
  if (!d_arena || !out) return LS_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(d_arena) & 255) != 0) return LS_ERR_INVALID_ARG;
  const ls::Layout y = ls::make_layout(*cfg);
  if (arena_bytes < size_t(y.total)) return LS_ERR_SHAPE;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LS_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LS_ERR_CUDA;
  if (cudaMemsetAsync(d_arena, 0, size_t(y.total), stream) != cudaSuccess) return LS_ERR_CUDA;

  ls_state* st = new (std::nothrow) ls_state;
  if (!st) return LS_ERR_INVALID_ARG;
  std::memset(static_cast<void*>(st), 0, sizeof(ls_state));
  st->cfg = *cfg;
  st->lay = y;
  st->arena = d_arena;
  st->device = dev;
  st->sms = sms;
  char* base = static_cast<char*>(d_arena);
  ls::Dev& p = st->dev;
  p.b = cfg->batch; p.L = cfg->n_layers; p.Hkv = cfg->n_kv_heads; p.Hq = cfg->n_q_heads;
  p.D = cfg->head_dim; p.hidden = cfg->hidden; p.B = cfg->block; p.W = cfg->window;
  p.nsc = cfg->n_scales; p.slots = cfg->slots_per_scale; p.R = y.R; p.dtype = cfg->dtype;
  p.out_f32 = (cfg->flags & LS_FLAG_OUT_F32) ? 1 : 0;
  for (int k = 0; k < LS_MAX_SCALES; ++k) p.scales[k] = k < cfg->n_scales ? cfg->scales[k] : 1;
  p.counters = reinterpret_cast<int64_t*>(base + y.counters);
  p.err = reinterpret_cast<int32_t*>(base + y.error);
  p.arrive = reinterpret_cast<int32_t*>(base + y.sync);
  p.kv = base + y.kv;
  p.seg = reinterpret_cast<float*>(base + y.seg);
  p.part = reinterpret_cast<float*>(base + y.part);
  p.glob = reinterpret_cast<float*>(base + y.glob);
  p.boundary = base + y.boundary;
  p.samp_count = reinterpret_cast<int32_t*>(base + y.sample);
  p.samp_part = reinterpret_cast<float*>(base + y.sample + int64_t(cfg->batch) * 4);
  p.samp_seg = p.samp_part + int64_t(cfg->batch) * ls::kSampleMaxChunks;
  p.pro_part = reinterpret_cast<float*>(base + y.prologue);
  p.pro_count = reinterpret_cast<int32_t*>(base + y.prologue + int64_t(ls::kProMaxSlots) * ls::kProTileN *
                                                                       ls::prologue_boundary_rows(cfg->batch) * 4);

  st->use_tc = 0;
  if (!(cfg->flags & LS_FLAG_FORCE_SIMT) && ls::tc_supported(p)) {
    const int r = ls::tc_prepare(p, &st->tc);
    if (r != LS_OK) { delete st; return r; }
    st->use_tc = 1;
  } else if (!ls::simt_supported(p)) {
    delete st;
    return LS_ERR_UNSUPPORTED;
  }
  *out = st;
  return LS_OK;
}

size_t ls_prefill_workspace_bytes(const ls_config* cfg, int64_t row_begin, int64_t row_end) {
  if (validate(cfg) != LS_OK || row_begin < 0 || row_end < row_begin) return 0;
  return ls::prefill_workspace_bytes(*cfg, row_begin, row_end);
}

int ls_prefill_summary(ls_state* st, const void* d_k, const void* d_v, int64_t plane_stride,
                       int64_t row_stride, const int64_t* d_prefix_len, int64_t row_begin,
                       int64_t row_end, const void* d_last_hidden, void* d_workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
  if (!st || !d_prefix_len) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  const ls_config& c = st->cfg;
  if (row_begin < 0 || row_end < row_begin) return LS_ERR_INVALID_ARG;
  if (row_begin % c.scales[c.n_scales - 1] != 0) return LS_ERR_SHAPE;
  const int64_t rowElems = int64_t(c.n_kv_heads) * c.head_dim;
  if (row_end > row_begin) {
    if (!d_k || !d_v || !d_workspace) return LS_ERR_INVALID_ARG;
    if (row_stride < rowElems || row_stride % 8 != 0 || plane_stride % 8 != 0) return LS_ERR_SHAPE;
    if (plane_stride < (row_end - row_begin) * row_stride && c.batch * c.n_layers > 1)
      return LS_ERR_SHAPE;
    if (!aligned16(d_k) || !aligned16(d_v) || !aligned16(d_workspace)) return LS_ERR_INVALID_ARG;
    if (workspace_bytes < ls::prefill_workspace_bytes(c, row_begin, row_end)) return LS_ERR_SHAPE;
  }
  if (d_last_hidden && !aligned16(d_last_hidden)) return LS_ERR_INVALID_ARG;
  return cuda_status(ls::launch_prefill(st->dev, c, d_k, d_v, plane_stride, row_stride,
                                        d_prefix_len, row_begin, row_end, d_last_hidden,
                                        d_workspace, st->sms, stream));
}

int ls_prefill_summary_noalloc(ls_state* st, const void* d_k, const void* d_v, int64_t plane_stride,
                               int64_t row_stride, const int64_t* d_prefix_len, int64_t row_begin,
                               int64_t row_end, const void* d_last_hidden, cudaStream_t stream) {
  if (!st || !d_prefix_len) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  const ls_config& c = st->cfg;
  if (row_begin < 0 || row_end < row_begin) return LS_ERR_INVALID_ARG;
  if (row_begin % c.scales[c.n_scales - 1] != 0) return LS_ERR_SHAPE;
  const int64_t rowElems = int64_t(c.n_kv_heads) * c.head_dim;
  if (row_end > row_begin) {
    if (!d_k || !d_v) return LS_ERR_INVALID_ARG;
    if (row_stride < rowElems || row_stride % 8 != 0 || plane_stride % 8 != 0) return LS_ERR_SHAPE;
    if (plane_stride < (row_end - row_begin) * row_stride && c.batch * c.n_layers > 1)
      return LS_ERR_SHAPE;
    if (!aligned16(d_k) || !aligned16(d_v)) return LS_ERR_INVALID_ARG;
  }
  if (d_last_hidden && !aligned16(d_last_hidden)) return LS_ERR_INVALID_ARG;
  if (ls::prefill_workspace_bytes(c, row_begin, row_end) > ls::noalloc_scratch_bytes())
    return LS_ERR_SCRATCH_LIMIT;
  void* ws = nullptr;
  if (ls::noalloc_scratch(st->device, &ws) != cudaSuccess) return LS_ERR_CUDA;
  return cuda_status(ls::launch_prefill(st->dev, c, d_k, d_v, plane_stride, row_stride, d_prefix_len,
                                        row_begin, row_end, d_last_hidden, ws, st->sms, stream));
}

int ls_prefill_paged(ls_state* st, const ls_paged_kv* h_kv, const int64_t* d_prefix_len, int64_t row_begin,
                     int64_t row_end, const void* d_last_hidden, void* d_workspace, size_t workspace_bytes,
                     cudaStream_t stream) {
  if (!st || !d_prefix_len) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  const ls_config& c = st->cfg;
  if (row_begin < 0 || row_end < row_begin) return LS_ERR_INVALID_ARG;
  if (row_begin % c.scales[c.n_scales - 1] != 0) return LS_ERR_SHAPE;
  if (row_end > row_begin) {
    const int v = validate_paged(c, h_kv);
    if (v != LS_OK) return v;
  }
  if (d_last_hidden && !aligned16(d_last_hidden)) return LS_ERR_INVALID_ARG;
  const size_t need = ls::prefill_workspace_bytes(c, row_begin, row_end);
  void* ws = d_workspace;
  if (ws) {
    if (!aligned16(ws)) return LS_ERR_INVALID_ARG;
    if (workspace_bytes < need) return LS_ERR_SHAPE;
  } else {  // the library's fixed scratch
    if (need > ls::noalloc_scratch_bytes()) return LS_ERR_SCRATCH_LIMIT;
    if (ls::noalloc_scratch(st->device, &ws) != cudaSuccess) return LS_ERR_CUDA;
  }
  static const ls_paged_kv kNone{};
  return cuda_status(ls::launch_prefill_paged(st->dev, c, row_end > row_begin ? *h_kv : kNone, d_prefix_len,
                                              row_begin, row_end, d_last_hidden, ws, st->sms, stream));
}

int ls_commit_round_paged(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                          const ls_paged_kv* h_kv, const void* d_verify_hidden, int32_t* d_accept_len,
                          int32_t* d_next_token, cudaStream_t stream) {
  if (!st || !d_draft_ids || !d_target_ids || !d_verify_hidden || !d_accept_len || !d_next_token)
    return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  const int v = validate_paged(st->cfg, h_kv);
  if (v != LS_OK) return v;
  if (!aligned16(d_verify_hidden)) return LS_ERR_INVALID_ARG;
  return cuda_status(ls::launch_commit_paged(st->dev, d_draft_ids, d_target_ids, *h_kv, d_verify_hidden,
                                             d_accept_len, d_next_token, nullptr, stream));
}

int ls_commit_accepted_paged(ls_state* st, const int32_t* d_accept_len, const ls_paged_kv* h_kv,
                             const void* d_verify_hidden, cudaStream_t stream) {
  if (!st || !d_accept_len || !d_verify_hidden) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  const int v = validate_paged(st->cfg, h_kv);
  if (v != LS_OK) return v;
  if (!aligned16(d_verify_hidden)) return LS_ERR_INVALID_ARG;
  return cuda_status(ls::launch_commit_paged(st->dev, nullptr, nullptr, *h_kv, d_verify_hidden, nullptr, nullptr,
                                             d_accept_len, stream));
}

int ls_commit_round(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids,
                    const void* d_verify_k, const void* d_verify_v, const void* d_verify_hidden,
                    int32_t* d_accept_len, int32_t* d_next_token, cudaStream_t stream) {
  if (!st || !d_draft_ids || !d_target_ids || !d_verify_k || !d_verify_v || !d_verify_hidden ||
      !d_accept_len || !d_next_token)
    return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  if (!aligned16(d_verify_k) || !aligned16(d_verify_v) || !aligned16(d_verify_hidden))
    return LS_ERR_INVALID_ARG;
  return cuda_status(ls::launch_commit(st->dev, d_draft_ids, d_target_ids, d_verify_k, d_verify_v,
                                       d_verify_hidden, d_accept_len, d_next_token, nullptr, stream));
}

int ls_accept_sampled(ls_state* st, const int32_t* d_draft_ids, const float* d_draft_probs,
                      const float* d_target_probs, int32_t vocab, const float* d_uniforms, int32_t* d_accept_len,
                      int32_t* d_next_token, cudaStream_t stream) {
  if (!st || !d_draft_ids || !d_draft_probs || !d_target_probs || !d_uniforms || !d_accept_len || !d_next_token)
    return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  if (vocab < 4 || vocab % 4 != 0) return LS_ERR_SHAPE;
  if (vocab > ls::kSampleChunk * ls::kSampleMaxChunks) return LS_ERR_UNSUPPORTED;
  if (!aligned16(d_draft_probs) || !aligned16(d_target_probs)) return LS_ERR_INVALID_ARG;
  const int r = cuda_status(ls::launch_sample(st->dev, d_draft_ids, d_draft_probs, d_target_probs, vocab, d_uniforms,
                                              d_accept_len, d_next_token, stream));
  if (r == LS_OK) mark_settled(st, stream);
  return r;
}

int ls_draft_prologue(const ls_state* st, const void* d_w_kv, const void* d_w_q, const void* d_x, void* d_bkv,
                      void* d_q, cudaStream_t stream) {
  if (!st || !d_w_kv || !d_w_q || !d_x || !d_bkv || !d_q) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  if (!ls::prologue_supported(st->dev)) return LS_ERR_UNSUPPORTED;
  if (!aligned16(d_w_kv) || !aligned16(d_w_q) || !aligned16(d_x) || !aligned16(d_bkv) || !aligned16(d_q))
    return LS_ERR_INVALID_ARG;
  const cudaError_t e = ls::launch_prologue(st->dev, d_w_kv, d_w_q, d_x, d_bkv, d_q, st->sms, stream);
  if (e == cudaSuccess) mark_settled(st, stream);
  return e == cudaErrorNotSupported ? LS_ERR_UNSUPPORTED : cuda_status(e);
}

int ls_commit_accepted(ls_state* st, const int32_t* d_accept_len, const void* d_verify_k, const void* d_verify_v,
                       const void* d_verify_hidden, cudaStream_t stream) {
  if (!st || !d_accept_len || !d_verify_k || !d_verify_v || !d_verify_hidden) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  if (!aligned16(d_verify_k) || !aligned16(d_verify_v) || !aligned16(d_verify_hidden)) return LS_ERR_INVALID_ARG;
  return cuda_status(ls::launch_commit(st->dev, nullptr, nullptr, d_verify_k, d_verify_v, d_verify_hidden, nullptr,
                                       nullptr, d_accept_len, stream));
}

int ls_draft_attend(const ls_state* st, int32_t layer_begin, int32_t layer_count, const void* d_q,
                    const void* d_boundary_k, const void* d_boundary_v, int64_t boundary_stride,
                    float softmax_scale, void* d_out, cudaStream_t stream) {
  return ls_draft_attend_views(st, layer_begin, layer_count, d_q, d_boundary_k, d_boundary_v, boundary_stride,
                               softmax_scale, LS_VIEW_ALL, d_out, stream);
}

int ls_draft_attend_views(const ls_state* st, int32_t layer_begin, int32_t layer_count, const void* d_q,
                          const void* d_boundary_k, const void* d_boundary_v, int64_t boundary_stride,
                          float softmax_scale, int32_t views, void* d_out, cudaStream_t stream) {
  if (!st || !d_q || !d_boundary_k || !d_boundary_v || !d_out) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  const bool inputs_ready = (views & LS_ATTEND_INPUTS_READY) != 0;
  views &= ~LS_ATTEND_INPUTS_READY;
  if (views == 0 || (views & ~LS_VIEW_ALL)) return LS_ERR_INVALID_ARG;
  const ls_config& c = st->cfg;
  if (layer_begin < 0 || layer_count < 1 || layer_begin + layer_count > c.n_layers)
    return LS_ERR_INVALID_ARG;
  if (boundary_stride < int64_t(c.n_kv_heads) * c.head_dim || boundary_stride % 8 != 0)
    return LS_ERR_SHAPE;
  if (!(softmax_scale > 0.0f) || softmax_scale == INFINITY) return LS_ERR_INVALID_ARG;
  if (!aligned16(d_q) || !aligned16(d_out) || !aligned16(d_boundary_k) || !aligned16(d_boundary_v))
    return LS_ERR_INVALID_ARG;
  if (st->use_tc) {
    // inside a stream capture the order of later replays is not known: no early loads
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess) return LS_ERR_CUDA;
    const bool settled = st->views_settled && st->settled_stream == stream && cap == cudaStreamCaptureStatusNone;
    const ls::AttendLaunch mode = settled ? (inputs_ready ? ls::kAttendFree : ls::kAttendViewsSettled)
                                          : (inputs_ready ? ls::kAttendAfterCommit : ls::kAttendPlain);
    const int r = cuda_status(ls::launch_attend_tc(st->dev, st->tc, layer_begin, layer_count, d_q, d_boundary_k,
                                                   d_boundary_v, boundary_stride, softmax_scale, views, d_out,
                                                   st->sms, mode, inputs_ready, stream));
    if (r == LS_OK) mark_settled(st, stream);
    return r;
  }
  return cuda_status(ls::launch_attend_simt(st->dev, layer_begin, layer_count, d_q, d_boundary_k,
                                            d_boundary_v, boundary_stride, softmax_scale, views, d_out,
                                            stream));
}

int ls_round(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids, const void* d_verify_k,
             const void* d_verify_v, const void* d_verify_hidden, int32_t* d_accept_len, int32_t* d_next_token,
             const void* d_q, int64_t boundary_k_offset, int64_t boundary_v_offset, float softmax_scale,
             void* d_out, cudaStream_t stream) {
  if (!st || !d_draft_ids || !d_target_ids || !d_verify_k || !d_verify_v || !d_verify_hidden || !d_accept_len ||
      !d_next_token || !d_q || !d_out)
    return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  const int rc = round_checks(st, boundary_k_offset, boundary_v_offset, softmax_scale, d_q, d_out);
  if (rc != LS_OK) return rc;
  int r = ls_commit_round(st, d_draft_ids, d_target_ids, d_verify_k, d_verify_v, d_verify_hidden, d_accept_len,
                          d_next_token, stream);
  if (r != LS_OK) return r;
  return round_attend(st, d_q, boundary_k_offset, boundary_v_offset, softmax_scale, d_out, stream);
}

int ls_round_paged(ls_state* st, const int32_t* d_draft_ids, const int32_t* d_target_ids, const ls_paged_kv* h_kv,
                   const void* d_verify_hidden, int32_t* d_accept_len, int32_t* d_next_token, const void* d_q,
                   int64_t boundary_k_offset, int64_t boundary_v_offset, float softmax_scale, void* d_out,
                   cudaStream_t stream) {
  if (!st || !d_q || !d_out) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  int r = round_checks(st, boundary_k_offset, boundary_v_offset, softmax_scale, d_q, d_out);
  if (r != LS_OK) return r;
  r = ls_commit_round_paged(st, d_draft_ids, d_target_ids, h_kv, d_verify_hidden, d_accept_len, d_next_token, stream);
  if (r != LS_OK) return r;
  return round_attend(st, d_q, boundary_k_offset, boundary_v_offset, softmax_scale, d_out, stream);
}

}  // extern "C"

namespace {
int round_attend(ls_state* st, const void* d_q, int64_t boundary_k_offset, int64_t boundary_v_offset,
                 float softmax_scale, void* d_out, cudaStream_t stream) {
  const ls_config& c = st->cfg;
  const char* bnd = static_cast<const char*>(st->dev.boundary);
  const int64_t e = st->lay.elem;
  if (st->use_tc) {  // the attention kernel is scheduled while the commit runs
    const int r = cuda_status(ls::launch_attend_tc(st->dev, st->tc, 0, c.n_layers, d_q, bnd + boundary_k_offset * e,
                                                   bnd + boundary_v_offset * e, c.hidden, softmax_scale, LS_VIEW_ALL,
                                                   d_out, st->sms, ls::kAttendAfterCommit, false, stream));
    if (r == LS_OK) mark_settled(st, stream);
    return r;
  }
  return ls_draft_attend(st, 0, c.n_layers, d_q, bnd + boundary_k_offset * e, bnd + boundary_v_offset * e, c.hidden,
                         softmax_scale, d_out, stream);
}
}  // namespace

extern "C" {

int ls_round_overlaps(const ls_state* st) { return st && st->use_tc ? 1 : 0; }

int ls_attend_uses_tensor_cores(const ls_state* st) { return st && st->use_tc ? 1 : 0; }

int ls_read_state(const ls_state* st, void* h_dst, size_t bytes, cudaStream_t stream) {
  if (!st || !h_dst) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  if (bytes > size_t(st->lay.total)) return LS_ERR_SHAPE;
  if (cudaMemcpyAsync(h_dst, st->arena, bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess)
    return LS_ERR_CUDA;
  return cuda_status(cudaStreamSynchronize(stream));
}

int ls_get_error(const ls_state* st, int32_t* h_code) {
  if (!st || !h_code) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return LS_ERR_CUDA;
  if (cudaMemcpy(h_code, st->dev.err, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LS_ERR_CUDA;
  if (*h_code & LS_DEVERR_WAIT_TIMEOUT) return LS_ERR_DEVICE_TIMEOUT;
  return *h_code ? LS_ERR_DEVICE : LS_OK;
}

int ls_clear_error(ls_state* st, cudaStream_t stream) {
  if (!st) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  st->views_settled = 0;  // this call writes the views
  // the error word, and the arrival counts a call that gave up part-way may have left
  // (they are zero between completed calls): the commit's, the sampler's, the projections'
  const ls::Layout& y = st->lay;
  const ls_config& c = st->cfg;
  char* base = static_cast<char*>(st->arena);
  if (cudaMemsetAsync(base + y.error, 0, 16, stream) != cudaSuccess) return LS_ERR_CUDA;
  if (cudaMemsetAsync(base + y.sync, 0, size_t(c.batch) * c.n_layers * 4, stream) != cudaSuccess) return LS_ERR_CUDA;
  if (cudaMemsetAsync(base + y.sample, 0, size_t(c.batch) * 4, stream) != cudaSuccess) return LS_ERR_CUDA;
  if (y.total > y.prologue &&
      cudaMemsetAsync(st->dev.pro_count, 0, size_t(ls::kProMaxGrid) * 4, stream) != cudaSuccess)
    return LS_ERR_CUDA;
  return LS_OK;
}

int ls_check_wait_timeout(ls_state* st, uint32_t polls, cudaStream_t stream) {
  if (!st || polls == 0 || polls > ls::kWaitLimit) return LS_ERR_INVALID_ARG;
  if (!on_state_device(st)) return LS_ERR_INVALID_ARG;
  const int r = cuda_status(ls::launch_wait_timeout(st->dev, polls, stream));
  if (r == LS_OK) mark_settled(st, stream);
  return r;
}

void ls_destroy_state(ls_state* st) { delete st; }

}  // extern "C"
