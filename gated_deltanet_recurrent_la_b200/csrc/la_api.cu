// la_api.cu -- the extern "C" entry points of liblastate.so (declared and documented in
// include/la_state.h): argument validation on the host, then one kernel launch on the
// caller's stream.  Nothing here allocates, frees or synchronizes.
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <unordered_set>
#include <utility>

#include <cuda_runtime.h>

#include "la_internal.h"
#include "la_state.h"
#include "la_device.cuh"

namespace la {

namespace {

thread_local int32_t g_last_cuda_error = 0;
// failure-path test hooks (la_debug_*): the wait limit of the decode step's pipeline waits,
// and a one-shot request to withhold one tile's arrival in the next decode step of the thread
thread_local uint64_t g_wait_ns = 0;       // 0: the default limit
thread_local int64_t g_withhold_tile = -1;

constexpr int kMaxDevices = 128;
int g_sm_count[kMaxDevices] = {0};
std::mutex g_mutex;
std::map<std::pair<const void*, int>, int> g_per_sm;

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

}  // namespace

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 0;
  int n = __atomic_load_n(&g_sm_count[dev], __ATOMIC_ACQUIRE);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    __atomic_store_n(&g_sm_count[dev], n, __ATOMIC_RELEASE);
  }
  return n;
}

int prepare_kernel(const void* func, int threads, int smem_bytes) {
  const int dev = current_device();
  if (dev < 0) return 0;
  std::lock_guard<std::mutex> lock(g_mutex);
  auto key = std::make_pair(func, dev);
  auto it = g_per_sm.find(key);
  if (it != g_per_sm.end()) return it->second;
  if (smem_bytes > 48 * 1024 &&
      cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
    return 0;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, func, threads, smem_bytes) != cudaSuccess) return 0;
  g_per_sm[key] = n;
  return n;
}

}  // namespace la

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_bytes(int32_t dt) { return dt == LA_F32 ? 4 : dt == LA_BF16 ? 2 : 0; }

bool shape_ok(const la_shape& s) {
  return s.n_qk_heads > 0 && s.n_v_heads > 0 && s.d_k > 0 && s.d_v > 0 && s.n_v_heads % s.n_qk_heads == 0;
}

bool same_shape(const la_shape& a, const la_shape& b) {
  return a.n_qk_heads == b.n_qk_heads && a.n_v_heads == b.n_v_heads && a.d_k == b.d_k && a.d_v == b.d_v;
}

la_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return LA_OK;
  la::g_last_cuda_error = static_cast<int32_t>(e);
  return LA_ERR_CUDA;
}

bool uses_gate(la_rule r) { return r == LA_RULE_GATED || r == LA_RULE_GATED_DELTA || r == LA_RULE_KDA; }
bool uses_beta(la_rule r) { return r == LA_RULE_DELTA || r == LA_RULE_GATED_DELTA || r == LA_RULE_KDA; }
// the rules whose chunked prefill has an intra-chunk launch (the two-launch form's workspace):
// the delta corrections of the delta rules, and kda's decay-scaled operands
bool chunk_inverse(la_rule r) { return r == LA_RULE_DELTA || r == LA_RULE_GATED_DELTA || r == LA_RULE_KDA; }
size_t chunk_ws_bytes(la_rule r, int64_t total_tokens, int64_t n_seqs, int64_t n_v_heads) {
  if (r == LA_RULE_KDA) return la::chunk_kda_workspace_bytes(total_tokens, n_seqs, n_v_heads);
  return chunk_inverse(r) ? la::chunk_workspace_bytes(total_tokens, n_seqs, n_v_heads) : 0;
}
// the gate array's alignment: kda's per-channel decays are moved in 16-byte pieces
size_t gate_align(la_rule r) { return r == LA_RULE_KDA ? 16 : 4; }

// Query-group direction: k has one head per state head (shape.n_qk_heads == n_v_heads)
// and n_q_heads query heads are read in groups of n_q_heads / n_v_heads <= 8.
la_status query_group(const la_shape& s, int32_t n_q_heads, int32_t* group) {
  if (n_q_heads <= 0 || s.n_qk_heads != s.n_v_heads || n_q_heads % s.n_v_heads) return LA_ERR_SHAPE;
  if (n_q_heads / s.n_v_heads > la::kMaxQueryGroup) return LA_ERR_UNSUPPORTED;
  *group = n_q_heads / s.n_v_heads;
  return LA_OK;
}

// q8 pools: d_v a multiple of the 32-column group, (d_k, d_v) one of the q8 tile shapes,
// an even number of BF16 channels of at most d_k / 4, and a channel mask.
bool q8_shape_ok(const la_shape& s) {
  return (s.d_k == 64 && s.d_v == 64) || (s.d_k == 128 && s.d_v == 64) || (s.d_k == 128 && s.d_v == 128);
}

la_status check_pool(const la_pool* p) {
  if (!p || !p->data) return LA_ERR_NULL;
  if (p->n_slots < 0 || !shape_ok(p->shape)) return LA_ERR_SHAPE;
  if (p->dtype == LA_Q8) {
    if (!q8_shape_ok(p->shape)) return LA_ERR_UNSUPPORTED;
    if (p->n_hp < 0 || p->n_hp % 2 || p->n_hp > p->shape.d_k / 4) return LA_ERR_SHAPE;
    if (!p->hp_mask) return LA_ERR_NULL;
    if (!aligned(p->hp_mask, 4)) return LA_ERR_ALIGN;
  } else if (!elem_bytes(p->dtype)) {
    return LA_ERR_UNSUPPORTED;
  }
  if (!aligned(p->data, 16)) return LA_ERR_ALIGN;
  return LA_OK;
}

// Bytes of one slot of a (checked) pool.
int64_t slot_bytes(const la_pool* p) {
  const la_shape& s = p->shape;
  if (p->dtype == LA_Q8) return (int64_t)s.n_v_heads * la::q8_tile_bytes(s.d_k, s.d_v, p->n_hp);
  return (int64_t)s.n_v_heads * s.d_k * s.d_v * elem_bytes(p->dtype);
}

}  // namespace

extern "C" {

size_t la_state_bytes(const la_shape* shape, la_dtype dtype) {
  if (!shape || !shape_ok(*shape) || !elem_bytes(dtype)) return 0;
  return (size_t)shape->n_v_heads * (size_t)shape->d_k * (size_t)shape->d_v * (size_t)elem_bytes(dtype);
}

int la_shape_supported(int32_t d_k, int32_t d_v) {
  return (d_k == 16 && d_v == 16) || (d_k == 64 && d_v == 64) || (d_k == 128 && d_v == 64) ||
         (d_k == 128 && d_v == 128);
}

// n_q_heads == 0: the default head direction; > 0: the query-group direction.  conv: the
// short causal convolution ahead of the step (q, k, v are then its inputs), or NULL.
static la_status step_impl(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                           const int32_t* write_slot, int32_t B, int32_t n_q_heads, const void* q, const void* k,
                           const void* v, la_dtype io, const float* g, const float* beta, float scale, void* o,
                           int32_t* err_word, void* stream, const la_conv* conv = nullptr) {
  if (rule < LA_RULE_LINEAR || rule > LA_RULE_KDA) return LA_ERR_UNSUPPORTED;
  if (!err_word) return LA_ERR_NULL;
  if (B < 0) return LA_ERR_SHAPE;
  la_status st = check_pool(src);
  if (st != LA_OK) return st;
  if ((st = check_pool(dst)) != LA_OK) return st;
  int32_t q_group = 1;
  if (n_q_heads != 0 && (st = query_group(src->shape, n_q_heads, &q_group)) != LA_OK) return st;
  if (B == 0) return LA_OK;
  if (!q || !k || !v || !o) return LA_ERR_NULL;
  if (uses_gate(rule) && !g) return LA_ERR_NULL;
  if (uses_beta(rule) && !beta) return LA_ERR_NULL;
  if (!same_shape(src->shape, dst->shape)) return LA_ERR_SHAPE;
  if (src->dtype != dst->dtype || !elem_bytes(io)) return LA_ERR_UNSUPPORTED;
  if (!la_shape_supported(src->shape.d_k, src->shape.d_v)) return LA_ERR_UNSUPPORTED;
  const bool q8 = src->dtype == LA_Q8;
  if (q8 && n_q_heads != 0) return LA_ERR_UNSUPPORTED;
  if (q8 && src->n_hp != dst->n_hp) return LA_ERR_SHAPE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(g, gate_align(rule)) ||
      !aligned(beta, 4) || !aligned(read_slot, 4) || !aligned(write_slot, 4) || !aligned(err_word, 4))
    return LA_ERR_ALIGN;
  if ((!read_slot && B > src->n_slots) || (!write_slot && B > dst->n_slots)) return LA_ERR_SHAPE;
  if ((int64_t)B * src->shape.n_v_heads > INT32_MAX) return LA_ERR_SHAPE;

  const la_shape& s = src->shape;
  if (conv) {
    if (q8) return LA_ERR_UNSUPPORTED;
    if (conv->width < 2 || conv->width > la::kMaxConvWidth) return LA_ERR_UNSUPPORTED;
    if (!conv->w_q || !conv->w_k || !conv->w_v || !conv->hist_src || !conv->hist_dst) return LA_ERR_NULL;
    if (!aligned(conv->w_q, 16) || !aligned(conv->w_k, 16) || !aligned(conv->w_v, 16) || !aligned(conv->hist_src, 16) ||
        !aligned(conv->hist_dst, 16))
      return LA_ERR_ALIGN;
  }
  la::StepLaunchFn fn = nullptr;
  if (conv)
    fn = (src->dtype == LA_F32) ? la::find_step_conv_f32(rule, s.d_k, s.d_v, io)
                                : la::find_step_conv_bf16(rule, s.d_k, s.d_v, io);
  else if (q8)
    fn = la::find_step_q8(rule, s.d_k, s.d_v, io);
  else if (n_q_heads == 0)
    fn = (src->dtype == LA_F32) ? la::find_step_f32(rule, s.d_k, s.d_v, io) : la::find_step_bf16(rule, s.d_k, s.d_v, io);
  else
    fn = (src->dtype == LA_F32) ? la::find_step_qgroups_f32(rule, s.d_k, s.d_v, io)
                                : la::find_step_qgroups_bf16(rule, s.d_k, s.d_v, io);
  if (!fn) return LA_ERR_UNSUPPORTED;
  la::StepParams p{};
  p.src = src->data;
  p.src_slots = src->n_slots;
  p.dst = dst->data;
  p.dst_slots = dst->n_slots;
  p.read_slot = read_slot;
  p.write_slot = write_slot;
  p.B = B;
  p.n_qk_heads = s.n_qk_heads;
  p.n_v_heads = s.n_v_heads;
  p.q_group = q_group;
  p.n_hp = q8 ? src->n_hp : 0;
  p.src_mask = q8 ? src->hp_mask : nullptr;
  p.dst_mask = q8 ? dst->hp_mask : nullptr;
  p.conv_w = conv ? conv->width : 0;
  p.conv_act = conv ? conv->activation : 0;
  p.conv_l2norm = conv ? conv->qk_l2norm : 0;
  p.conv_wq = conv ? conv->w_q : nullptr;
  p.conv_wk = conv ? conv->w_k : nullptr;
  p.conv_wv = conv ? conv->w_v : nullptr;
  p.conv_src = conv ? conv->hist_src : nullptr;
  p.conv_dst = conv ? conv->hist_dst : nullptr;
  p.q = q;
  p.k = k;
  p.v = v;
  p.g = uses_gate(rule) ? g : nullptr;
  p.beta = uses_beta(rule) ? beta : nullptr;
  p.scale = scale;
  p.o = o;
  p.err = err_word;
  p.wait_ns = la::g_wait_ns ? la::g_wait_ns : la::kWaitLimitNs;
  p.withhold = la::g_withhold_tile;
  la::g_withhold_tile = -1;  // one-shot
  return cuda_status(fn(p, static_cast<cudaStream_t>(stream)));
}

la_status la_state_step(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                        const int32_t* write_slot, int32_t B, const void* q, const void* k, const void* v,
                        la_dtype io, const float* g, const float* beta, float scale, void* o, int32_t* err_word,
                        void* stream) {
  return step_impl(rule, src, read_slot, dst, write_slot, B, 0, q, k, v, io, g, beta, scale, o, err_word, stream);
}

la_status la_state_step_conv(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                             const int32_t* write_slot, int32_t B, const la_conv* conv, const void* xq,
                             const void* xk, const void* xv, la_dtype io, const float* g, const float* beta,
                             float scale, void* o, int32_t* err_word, void* stream) {
  if (!conv) return LA_ERR_NULL;
  return step_impl(rule, src, read_slot, dst, write_slot, B, 0, xq, xk, xv, io, g, beta, scale, o, err_word, stream,
                   conv);
}

la_status la_state_step_qgroups(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                const int32_t* write_slot, int32_t B, int32_t n_q_heads, const void* q, const void* k,
                                const void* v, la_dtype io, const float* g, const float* beta, float scale, void* o,
                                int32_t* err_word, void* stream) {
  if (n_q_heads <= 0) return LA_ERR_SHAPE;
  return step_impl(rule, src, read_slot, dst, write_slot, B, n_q_heads, q, k, v, io, g, beta, scale, o, err_word,
                   stream);
}

static la_status scan_impl(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                           const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens, int32_t total_tokens,
                           const int32_t* seq_order, const void* q, const void* k, const void* v, la_dtype io,
                           const float* g, const float* beta, float scale, void* o, int32_t ckpt_every,
                           const int32_t* ckpt_cu, const int32_t* ckpt_slots, int32_t* err_word, void* stream,
                           bool chunked = false, int32_t n_q_heads = 0, const la_conv* conv = nullptr,
                           void* workspace = nullptr, size_t workspace_bytes = 0) {
  if (rule < LA_RULE_LINEAR || rule > LA_RULE_KDA) return LA_ERR_UNSUPPORTED;
  if (!err_word) return LA_ERR_NULL;
  if (n_seqs < 0 || total_tokens < 0) return LA_ERR_SHAPE;
  la_status st = check_pool(dst);
  if (st != LA_OK) return st;
  int32_t q_group = 1;
  if (n_q_heads != 0 && (st = query_group(dst->shape, n_q_heads, &q_group)) != LA_OK) return st;
  if (read_slot) {
    if ((st = check_pool(src)) != LA_OK) return st;
    if (!same_shape(src->shape, dst->shape)) return LA_ERR_SHAPE;
  }
  if (n_seqs == 0) return LA_OK;
  if (!cu_seqlens) return LA_ERR_NULL;
  if (total_tokens > 0) {
    if (!q || !k || !v || !o) return LA_ERR_NULL;
    if (uses_gate(rule) && !g) return LA_ERR_NULL;
    if (uses_beta(rule) && !beta) return LA_ERR_NULL;
  }
  if (!elem_bytes(io)) return LA_ERR_UNSUPPORTED;
  const la_shape& s = dst->shape;
  if (!la_shape_supported(s.d_k, s.d_v)) return LA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(g, gate_align(rule)) ||
      !aligned(beta, 4) || !aligned(read_slot, 4) || !aligned(write_slot, 4) || !aligned(cu_seqlens, 4) ||
      !aligned(seq_order, 4) || !aligned(err_word, 4))
    return LA_ERR_ALIGN;
  if (!write_slot && n_seqs > dst->n_slots) return LA_ERR_SHAPE;
  if ((int64_t)n_seqs * s.n_v_heads > INT32_MAX) return LA_ERR_SHAPE;

  const bool q8 = dst->dtype == LA_Q8 || (read_slot && src->dtype == LA_Q8);
  // q8 pools on the chunked path: the one-launch form of the scalar-gate rules (query groups
  // included); on the token-serial scan not in the query-group direction
  if (q8 && ((n_q_heads != 0 && !chunked) || (chunked && (workspace || conv || rule == LA_RULE_KDA))))
    return LA_ERR_UNSUPPORTED;
  if (conv) {
    if (q8 || n_q_heads != 0 || ckpt_every > 0) return LA_ERR_UNSUPPORTED;
    if (conv->width < 2 || conv->width > la::kMaxConvWidth) return LA_ERR_UNSUPPORTED;
    if (!conv->w_q || !conv->w_k || !conv->w_v || !conv->hist_dst || (read_slot && !conv->hist_src))
      return LA_ERR_NULL;
    if (!aligned(conv->w_q, 4) || !aligned(conv->w_k, 4) || !aligned(conv->w_v, 4) || !aligned(conv->hist_src, 16) ||
        !aligned(conv->hist_dst, 16))
      return LA_ERR_ALIGN;
  }
  la::ScanLaunchFn fn = nullptr;
  if (conv && chunked) {
    if (s.d_k != 128 || s.d_v != 128 || io != LA_BF16) return LA_ERR_UNSUPPORTED;
    if (workspace) {
      if (!aligned(workspace, 16)) return LA_ERR_ALIGN;
      if (workspace_bytes < la::chunk_conv_workspace_bytes(total_tokens, s.n_v_heads)) return LA_ERR_SHAPE;
      fn = la::find_chunk_scan_conv_ws(rule);
    } else {
      fn = la::find_chunk_scan_conv(rule);
    }
  } else if (conv) {
    fn = (io == LA_F32) ? la::find_scan_conv_f32io(rule, s.d_k, s.d_v) : la::find_scan_conv_bf16io(rule, s.d_k, s.d_v);
  } else if (chunked && n_q_heads != 0) {
    // the query-group direction: the one-launch form of the scalar-gate rules, once per query
    if (s.d_k != 128 || s.d_v != 128 || io != LA_BF16) return LA_ERR_UNSUPPORTED;
    if (ckpt_every > 0 || workspace) return LA_ERR_UNSUPPORTED;
    fn = la::find_chunk_scan_qgroups(rule);
  } else if (chunked) {
    if (s.d_k != 128 || s.d_v != 128 || io != LA_BF16) return LA_ERR_UNSUPPORTED;
    // checkpoints fall on chunk boundaries, in the one-launch form
    if (ckpt_every > 0 && (ckpt_every % 64 != 0 || workspace)) return LA_ERR_UNSUPPORTED;
    if (workspace && chunk_inverse(rule)) {
      if (!aligned(workspace, 16)) return LA_ERR_ALIGN;
      if (workspace_bytes < chunk_ws_bytes(rule, total_tokens, n_seqs, s.n_v_heads)) return LA_ERR_SHAPE;
      fn = la::find_chunk_scan_ws(rule);
    } else {
      fn = la::find_chunk_scan(rule);
    }
  } else if (n_q_heads == 0) {
    fn = (io == LA_F32) ? la::find_scan_f32io(rule, s.d_k, s.d_v) : la::find_scan_bf16io(rule, s.d_k, s.d_v);
  } else {
    fn = (io == LA_F32) ? la::find_scan_qgroups_f32io(rule, s.d_k, s.d_v)
                        : la::find_scan_qgroups_bf16io(rule, s.d_k, s.d_v);
  }
  if (!fn) return LA_ERR_UNSUPPORTED;
  la::ScanParams p{};
  p.src = read_slot ? src->data : nullptr;
  p.src_slots = read_slot ? src->n_slots : 0;
  p.src_dtype = read_slot ? src->dtype : dst->dtype;
  p.read_slot = read_slot;
  p.dst = dst->data;
  p.dst_slots = dst->n_slots;
  p.dst_dtype = dst->dtype;
  p.write_slot = write_slot;
  p.n_seqs = n_seqs;
  p.cu_seqlens = cu_seqlens;
  p.total_tokens = total_tokens;
  p.seq_order = seq_order;
  p.n_qk_heads = s.n_qk_heads;
  p.n_v_heads = s.n_v_heads;
  p.q_group = q_group;
  p.src_n_hp = read_slot && src->dtype == LA_Q8 ? src->n_hp : 0;
  p.src_mask = read_slot && src->dtype == LA_Q8 ? src->hp_mask : nullptr;
  p.dst_n_hp = dst->dtype == LA_Q8 ? dst->n_hp : 0;
  p.dst_mask = dst->dtype == LA_Q8 ? dst->hp_mask : nullptr;
  p.q = q;
  p.k = k;
  p.v = v;
  p.g = uses_gate(rule) ? g : nullptr;
  p.beta = uses_beta(rule) ? beta : nullptr;
  p.scale = scale;
  p.o = o;
  p.err = err_word;
  p.ckpt_every = ckpt_every;
  p.ckpt_cu = ckpt_cu;
  p.ckpt_slots = ckpt_slots;
  p.workspace = workspace;
  if (conv) {
    p.conv_w = conv->width;
    p.conv_act = conv->activation;
    p.conv_l2norm = conv->qk_l2norm;
    p.conv_wq = conv->w_q;
    p.conv_wk = conv->w_k;
    p.conv_wv = conv->w_v;
    p.conv_src = conv->hist_src;
    p.conv_dst = conv->hist_dst;
  }
  return cuda_status(fn(p, static_cast<cudaStream_t>(stream)));
}

la_status la_state_scan(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                        const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens, int32_t total_tokens,
                        const int32_t* seq_order, const void* q, const void* k, const void* v, la_dtype io,
                        const float* g, const float* beta, float scale, void* o, int32_t* err_word, void* stream) {
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream);
}

la_status la_state_scan_chunked(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                                int32_t total_tokens, const int32_t* seq_order, const void* q, const void* k,
                                const void* v, la_dtype io, const float* g, const float* beta, float scale, void* o,
                                int32_t* err_word, void* stream) {
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, true);
}

size_t la_scan_chunked_workspace_bytes(int32_t total_tokens, int32_t n_seqs, int32_t n_v_heads) {
  return la::chunk_workspace_bytes(total_tokens, n_seqs, n_v_heads);
}

size_t la_scan_chunked_workspace_bytes_rule(la_rule rule, int32_t total_tokens, int32_t n_seqs,
                                            int32_t n_v_heads) {
  if (rule < LA_RULE_LINEAR || rule > LA_RULE_KDA) return 0;
  return chunk_ws_bytes(rule, total_tokens, n_seqs, n_v_heads);
}

la_status la_state_scan_chunked_ws(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                   const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                                   int32_t total_tokens, const int32_t* seq_order, const void* q, const void* k,
                                   const void* v, la_dtype io, const float* g, const float* beta, float scale,
                                   void* o, void* workspace, size_t workspace_bytes, int32_t* err_word,
                                   void* stream) {
  if (!workspace && n_seqs > 0 && chunk_inverse(rule)) return LA_ERR_NULL;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, true, 0, nullptr, workspace,
                   workspace_bytes);
}

la_status la_state_scan_chunked_noalloc(la_rule rule, const la_pool* src, const int32_t* read_slot,
                                        const la_pool* dst, const int32_t* write_slot, int32_t n_seqs,
                                        const int32_t* cu_seqlens, int32_t total_tokens, const int32_t* seq_order,
                                        const void* q, const void* k, const void* v, la_dtype io, const float* g,
                                        const float* beta, float scale, void* o, int32_t* err_word, void* stream) {
  size_t bytes = 0;
  void* ws = nullptr;
  const cudaError_t e = la::chunk_noalloc_workspace(&ws, &bytes);
  if (e != cudaSuccess) return cuda_status(e);
  return la_state_scan_chunked_ws(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order,
                                  q, k, v, io, g, beta, scale, o, ws, bytes, err_word, stream);
}

la_status la_state_scan_checkpointed(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                     const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                                     int32_t total_tokens, const int32_t* seq_order, const void* q, const void* k,
                                     const void* v, la_dtype io, const float* g, const float* beta, float scale,
                                     void* o, int32_t ckpt_every, const int32_t* ckpt_cu, const int32_t* ckpt_slots,
                                     int32_t* err_word, void* stream) {
  if (ckpt_every <= 0) return LA_ERR_SHAPE;
  if (n_seqs > 0 && (!ckpt_cu || !ckpt_slots)) return LA_ERR_NULL;
  if (!aligned(ckpt_cu, 4) || !aligned(ckpt_slots, 4)) return LA_ERR_ALIGN;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, err_word, stream);
}

la_status la_state_scan_chunked_checkpointed(la_rule rule, const la_pool* src, const int32_t* read_slot,
                                             const la_pool* dst, const int32_t* write_slot, int32_t n_seqs,
                                             const int32_t* cu_seqlens, int32_t total_tokens,
                                             const int32_t* seq_order, const void* q, const void* k, const void* v,
                                             la_dtype io, const float* g, const float* beta, float scale, void* o,
                                             int32_t ckpt_every, const int32_t* ckpt_cu, const int32_t* ckpt_slots,
                                             int32_t* err_word, void* stream) {
  if (ckpt_every <= 0) return LA_ERR_SHAPE;
  if (n_seqs > 0 && (!ckpt_cu || !ckpt_slots)) return LA_ERR_NULL;
  if (!aligned(ckpt_cu, 4) || !aligned(ckpt_slots, 4)) return LA_ERR_ALIGN;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, ckpt_every, ckpt_cu, ckpt_slots, err_word, stream, true);
}

la_status la_state_scan_conv(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                             const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                             int32_t total_tokens, const int32_t* seq_order, const la_conv* conv, const void* xq,
                             const void* xk, const void* xv, la_dtype io, const float* g, const float* beta,
                             float scale, void* o, int32_t* err_word, void* stream) {
  if (!conv) return LA_ERR_NULL;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, xq, xk, xv, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, false, 0, conv);
}

la_status la_state_scan_chunked_conv(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                     const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                                     int32_t total_tokens, const int32_t* seq_order, const la_conv* conv,
                                     const void* xq, const void* xk, const void* xv, la_dtype io, const float* g,
                                     const float* beta, float scale, void* o, int32_t* err_word, void* stream) {
  if (!conv) return LA_ERR_NULL;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, xq, xk, xv, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, true, 0, conv);
}

size_t la_scan_chunked_conv_workspace_bytes(int32_t total_tokens, int32_t n_v_heads) {
  return la::chunk_conv_workspace_bytes(total_tokens, n_v_heads);
}

la_status la_state_scan_chunked_conv_ws(la_rule rule, const la_pool* src, const int32_t* read_slot,
                                        const la_pool* dst, const int32_t* write_slot, int32_t n_seqs,
                                        const int32_t* cu_seqlens, int32_t total_tokens, const int32_t* seq_order,
                                        const la_conv* conv, const void* xq, const void* xk, const void* xv,
                                        la_dtype io, const float* g, const float* beta, float scale, void* o,
                                        void* workspace, size_t workspace_bytes, int32_t* err_word, void* stream) {
  if (!conv) return LA_ERR_NULL;
  if (!workspace && n_seqs > 0) return LA_ERR_NULL;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, xq, xk, xv, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, true, 0, conv, workspace,
                   workspace_bytes);
}

la_status la_state_scan_qgroups(la_rule rule, const la_pool* src, const int32_t* read_slot, const la_pool* dst,
                                const int32_t* write_slot, int32_t n_seqs, const int32_t* cu_seqlens,
                                int32_t total_tokens, const int32_t* seq_order, int32_t n_q_heads, const void* q,
                                const void* k, const void* v, la_dtype io, const float* g, const float* beta,
                                float scale, void* o, int32_t* err_word, void* stream) {
  if (n_q_heads <= 0) return LA_ERR_SHAPE;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, false, n_q_heads);
}

la_status la_state_scan_chunked_qgroups(la_rule rule, const la_pool* src, const int32_t* read_slot,
                                        const la_pool* dst, const int32_t* write_slot, int32_t n_seqs,
                                        const int32_t* cu_seqlens, int32_t total_tokens, const int32_t* seq_order,
                                        int32_t n_q_heads, const void* q, const void* k, const void* v, la_dtype io,
                                        const float* g, const float* beta, float scale, void* o, int32_t* err_word,
                                        void* stream) {
  if (n_q_heads <= 0) return LA_ERR_SHAPE;
  return scan_impl(rule, src, read_slot, dst, write_slot, n_seqs, cu_seqlens, total_tokens, seq_order, q, k, v, io,
                   g, beta, scale, o, 0, nullptr, nullptr, err_word, stream, true, n_q_heads);
}

static la_status pool_op(const la_pool* pool, int32_t n, const int32_t* src_slots, const int32_t* dst_slots,
                         const void* src_dense, void* dst_dense, int zero, int32_t* err_word, void* stream) {
  if (!err_word) return LA_ERR_NULL;
  if (n < 0) return LA_ERR_SHAPE;
  la_status st = check_pool(pool);
  if (st != LA_OK) return st;
  if (n == 0) return LA_OK;
  if (!aligned(src_slots, 4) || !aligned(dst_slots, 4) || !aligned(err_word, 4) || !aligned(src_dense, 16) ||
      !aligned(dst_dense, 16))
    return LA_ERR_ALIGN;
  la::PoolCopyParams p;
  p.slot_bytes = slot_bytes(pool);
  p.n = n;
  p.zero = zero;
  p.err = err_word;
  if (src_dense) {  // scatter: dense -> pool
    p.src = src_dense;
    p.src_index = nullptr;
    p.src_count = n;
    p.dst = pool->data;
    p.dst_index = dst_slots;
    p.dst_count = pool->n_slots;
  } else if (dst_dense) {  // gather: pool -> dense
    p.src = pool->data;
    p.src_index = src_slots;
    p.src_count = pool->n_slots;
    p.dst = dst_dense;
    p.dst_index = nullptr;
    p.dst_count = n;
  } else {  // copy or zero within the pool
    p.src = pool->data;
    p.src_index = src_slots;
    p.src_count = pool->n_slots;
    p.dst = pool->data;
    p.dst_index = dst_slots;
    p.dst_count = pool->n_slots;
  }
  return cuda_status(la::launch_pool_copy(p, static_cast<cudaStream_t>(stream)));
}

la_status la_state_pool_copy(const la_pool* pool, int32_t n, const int32_t* src_slots, const int32_t* dst_slots,
                             int32_t* err_word, void* stream) {
  if (n > 0 && (!src_slots || !dst_slots)) return LA_ERR_NULL;
  return pool_op(pool, n, src_slots, dst_slots, nullptr, nullptr, 0, err_word, stream);
}

la_status la_state_pool_gather(const la_pool* pool, int32_t n, const int32_t* slots, void* dense, int32_t* err_word,
                               void* stream) {
  if (n > 0 && (!slots || !dense)) return LA_ERR_NULL;
  return pool_op(pool, n, slots, nullptr, nullptr, dense, 0, err_word, stream);
}

la_status la_state_pool_scatter(const la_pool* pool, int32_t n, const int32_t* slots, const void* dense,
                                int32_t* err_word, void* stream) {
  if (n > 0 && (!slots || !dense)) return LA_ERR_NULL;
  return pool_op(pool, n, nullptr, slots, dense, nullptr, 0, err_word, stream);
}

la_status la_state_pool_zero(const la_pool* pool, int32_t n, const int32_t* slots, int32_t* err_word, void* stream) {
  if (n > 0 && !slots) return LA_ERR_NULL;
  return pool_op(pool, n, nullptr, slots, nullptr, nullptr, 1, err_word, stream);
}

static la_status q8_codec(const la_pool* pool, int32_t n, const int32_t* slots, float* dense, int encode,
                          int32_t* err_word, void* stream) {
  if (!err_word) return LA_ERR_NULL;
  if (n < 0) return LA_ERR_SHAPE;
  la_status st = check_pool(pool);
  if (st != LA_OK) return st;
  if (pool->dtype != LA_Q8) return LA_ERR_UNSUPPORTED;
  if (n == 0) return LA_OK;
  if (!slots || !dense) return LA_ERR_NULL;
  if (!aligned(slots, 4) || !aligned(dense, 16) || !aligned(err_word, 4)) return LA_ERR_ALIGN;
  la::Q8CodecParams p;
  p.pool = pool->data;
  p.n_slots = pool->n_slots;
  p.n_v_heads = pool->shape.n_v_heads;
  p.d_k = pool->shape.d_k;
  p.d_v = pool->shape.d_v;
  p.n_hp = pool->n_hp;
  p.mask = pool->hp_mask;
  p.slots = slots;
  p.n = n;
  p.dense = dense;
  p.encode = encode;
  p.err = err_word;
  return cuda_status(la::launch_q8_codec(p, static_cast<cudaStream_t>(stream)));
}

la_status la_state_pool_encode(const la_pool* pool, int32_t n, const int32_t* slots, const float* dense,
                               int32_t* err_word, void* stream) {
  return q8_codec(pool, n, slots, const_cast<float*>(dense), 1, err_word, stream);
}

la_status la_state_pool_decode(const la_pool* pool, int32_t n, const int32_t* slots, float* dense, int32_t* err_word,
                               void* stream) {
  return q8_codec(pool, n, slots, dense, 0, err_word, stream);
}

size_t la_pool_slot_bytes(const la_pool* pool) {
  if (check_pool(pool) != LA_OK) return 0;
  return (size_t)slot_bytes(pool);
}

la_status la_state_check_slots(int32_t B, const int32_t* read_slot_host, const int32_t* write_slot_host,
                               int32_t n_slots) {
  if (B < 0 || n_slots < 0) return LA_ERR_SHAPE;
  std::unordered_set<int32_t> writes;
  for (int32_t b = 0; b < B; ++b) {
    const int32_t r = read_slot_host ? read_slot_host[b] : b;
    const int32_t w = write_slot_host ? write_slot_host[b] : b;
    if (r < 0 || r >= n_slots || w < 0 || w >= n_slots) return LA_ERR_SHAPE;
    if (!writes.insert(w).second) return LA_ERR_ALIAS;
  }
  for (int32_t b = 0; b < B; ++b) {
    const int32_t r = read_slot_host ? read_slot_host[b] : b;
    const int32_t w = write_slot_host ? write_slot_host[b] : b;
    if (r != w && writes.count(r)) return LA_ERR_ALIAS;  // reads a slot another request overwrites
  }
  return LA_OK;
}

const char* la_status_str(la_status status) {
  switch (status) {
    case LA_OK: return "LA_OK";
    case LA_ERR_NULL: return "LA_ERR_NULL: a required pointer is NULL";
    case LA_ERR_SHAPE: return "LA_ERR_SHAPE: invalid or inconsistent sizes";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: shape, dtype or rule not supported";
    case LA_ERR_ALIGN: return "LA_ERR_ALIGN: pointer alignment";
    case LA_ERR_ALIAS: return "LA_ERR_ALIAS: slot preconditions violated";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: the CUDA runtime refused the launch";
  }
  return "unknown la_status";
}

int32_t la_last_cuda_error(void) { return la::g_last_cuda_error; }

void la_debug_set_wait_limit_us(uint32_t us) { la::g_wait_ns = (uint64_t)us * 1000u; }

void la_debug_withhold_step_tile(int32_t tile) { la::g_withhold_tile = tile < 0 ? -1 : tile; }

int32_t la_abi_version(void) { return LA_ABI_VERSION; }

}  // extern "C"
