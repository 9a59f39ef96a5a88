// C entry points of libosp.so: argument validation, error reporting and dispatch to the
// kernels.  Every check here runs on the host before anything is enqueued.

#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <initializer_list>
#include <mutex>
#include <set>
#include <utility>

#include "osp_internal.h"

namespace osp {

namespace {
thread_local char g_last_error[512] = "";

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned* g_status[kMaxDevices] = {};
cudaMemPool_t g_pool[kMaxDevices] = {};
std::atomic<int> g_sms[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int check_shape(const osp_shape* s, bool attention) {
  if (!s) return set_error(OSP_ERR_INVALID_ARG, "shape is NULL");
  if (s->B < 1 || s->text_len < 0 || s->T < 1 || s->H < 1 || s->W < 1 || s->heads < 1 || s->head_dim < 2)
    return set_error(OSP_ERR_INVALID_ARG, "bad shape: B=%d text_len=%d T=%d H=%d W=%d heads=%d head_dim=%d", s->B,
                     s->text_len, s->T, s->H, s->W, s->heads, s->head_dim);
  if (s->head_dim % 8)
    return set_error(OSP_ERR_UNSUPPORTED, "head_dim %d is not a multiple of 8", s->head_dim);
  const long long n = (long long)s->text_len + (long long)s->T * s->H * s->W;
  if (n > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "sequence length %lld too large", n);
  if (attention && s->head_dim != 64 && s->head_dim != 96 && s->head_dim != 128)
    return set_error(OSP_ERR_UNSUPPORTED, "attention head_dim %d not in {64, 96, 128}", s->head_dim);
  return OSP_OK;
}

int check_rope(const osp_rope* r, int head_dim) {
  if (!r) return set_error(OSP_ERR_INVALID_ARG, "rope is NULL");
  if (r->d_t < 0 || r->d_h < 0 || r->d_w < 0 || (r->d_t | r->d_h | r->d_w) & 1)
    return set_error(OSP_ERR_INVALID_ARG, "RoPE chunks must be even and >= 0 (got %d/%d/%d)", r->d_t, r->d_h,
                     r->d_w);
  if (r->d_t + r->d_h + r->d_w != head_dim)
    return set_error(OSP_ERR_INVALID_ARG, "RoPE split %d/%d/%d does not sum to head_dim %d", r->d_t, r->d_h,
                     r->d_w, head_dim);
  if (!(r->theta > 0.0) || !std::isfinite(r->theta))
    return set_error(OSP_ERR_INVALID_ARG, "RoPE theta must be finite and > 0");
  if (head_dim > 256) return set_error(OSP_ERR_UNSUPPORTED, "RoPE head_dim %d > 256", head_dim);
  return OSP_OK;
}

int check_skiparse(const osp_shape* s, int k, int mode, bool allow_text = false) {
  if (k < 1) return set_error(OSP_ERR_INVALID_ARG, "sparse ratio k=%d < 1", k);
  if (mode != OSP_SKIP_SINGLE && mode != OSP_SKIP_GROUP)
    return set_error(OSP_ERR_INVALID_ARG, "mode %d is neither OSP_SKIP_SINGLE nor OSP_SKIP_GROUP", mode);
  if (s->text_len != 0 && !allow_text)
    return set_error(OSP_ERR_UNSUPPORTED, "Skiparse gather / scatter take video tokens only (text_len=%d)",
                     s->text_len);
  const long long nv = (long long)s->T * s->H * s->W;
  const long long step = (mode == OSP_SKIP_SINGLE) ? k : (long long)k * k;
  if (nv % step)
    return set_error(OSP_ERR_DIVISIBILITY, "T*H*W=%lld is not a multiple of %lld", nv, step);
  return OSP_OK;
}
}  // namespace

int set_error(int code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
  return code;
}

int check_launch(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return set_error(OSP_ERR_CUDA, "%s launch failed: %s", what, cudaGetErrorString(e));
  return OSP_OK;
}

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  int n = g_sms[dev].load(std::memory_order_relaxed);
  if (!n) {
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    n = n > 0 ? n : 148;
    g_sms[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

unsigned* device_status_word() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) {
    set_error(OSP_ERR_CUDA, "no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status[dev]) {
    void* p = nullptr;
    if (cudaMalloc(&p, 256) != cudaSuccess || cudaMemset(p, 0, 256) != cudaSuccess) {
      set_error(OSP_ERR_CUDA, "status word allocation failed");
      return nullptr;
    }
    g_status[dev] = static_cast<unsigned*>(p);
  }
  return g_status[dev];
}

unsigned* device_status_word_if_present() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  return g_status[dev];
}

cudaMemPool_t workspace_pool() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_pool[dev]) {
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.handleTypes = cudaMemHandleTypeNone;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    // keep freed workspace cached in the pool instead of returning it at every synchronisation
    uint64_t keep = ~0ull;
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    g_pool[dev] = pool;
  }
  return g_pool[dev];
}

uint64_t wait_timeout_ns() {
  const char* e = getenv("OSP_WAIT_TIMEOUT_MS");
  const long long ms = e ? atoll(e) : 2000;
  return (uint64_t)(ms > 0 ? ms : 2000) * 1000000ull;
}

int split_kv_enabled() {
  const char* e = getenv("OSP_SPLIT_KV");
  return (e && e[0] == '0') ? 0 : 1;
}

int ensure_smem_attr(const void* func, int bytes, const char* name) {
  static std::mutex mu;
  static std::set<std::pair<int, const void*>> done;
  const int dev = current_device();
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({dev, func})) return OSP_OK;
  const cudaError_t e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess)
    return set_error(OSP_ERR_CUDA, "cudaFuncSetAttribute(%s, %d bytes of shared memory) failed: %s", name, bytes,
                     cudaGetErrorString(e));
  done.insert({dev, func});
  return OSP_OK;
}

unsigned bounds_check_divisor() {
  const char* e = getenv("OSP_DEBUG_BOUNDS_DIV");
  const long v = e ? strtol(e, nullptr, 10) : 1;
  return v >= 1 ? (unsigned)v : 1u;
}

int persist_mode() {
  const char* e = getenv("OSP_PERSIST");
  if (!e || !e[0]) return 1;
  return e[0] == '0' ? 0 : (e[0] == '2' ? 2 : 1);
}

int debug_withhold_q() {
  const char* e = getenv("OSP_DEBUG_WITHHOLD_Q");
  return (e && e[0] == '1') ? 1 : 0;
}

// Offsets of a packed batch: n + 1 host values, bounds[0] = 0, non-decreasing, total <= 2^30.
int check_bounds(const int32_t* b, int n, const char* what) {
  if (!b) return set_error(OSP_ERR_INVALID_ARG, "%s is NULL", what);
  if (b[0] != 0) return set_error(OSP_ERR_INVALID_ARG, "%s[0] = %d, must be 0", what, b[0]);
  for (int i = 0; i < n; ++i)
    if (b[i + 1] < b[i])
      return set_error(OSP_ERR_INVALID_ARG, "%s decreases at %d (%d -> %d)", what, i, b[i], b[i + 1]);
  if (b[n] > (1 << 30)) return set_error(OSP_ERR_UNSUPPORTED, "%s: %d rows is too many", what, b[n]);
  return OSP_OK;
}

}  // namespace osp

using namespace osp;

extern "C" {

const char* osp_get_last_error(void) { return g_last_error; }

int osp_version(void) { return 100; }

int osp_rope3d(const void* q, const void* k, void* q_out, void* k_out, const osp_shape* shape, const osp_rope* rope,
               void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, false);
  if (rc) return rc;
  if ((rc = check_rope(rope, shape->head_dim))) return rc;
  if (!q || !k || !q_out || !k_out) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return rope3d_launch(q, k, q_out, k_out, *shape, *rope, static_cast<cudaStream_t>(stream));
}

int osp_attn_full(const void* q, const void* k, const void* v, void* o, const osp_shape* shape, float softmax_scale,
                  void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return attention_launch(q, k, v, o, *shape, 0, 1, softmax_scale, static_cast<cudaStream_t>(stream));
}

int osp_attn_cross(const void* q, const void* k, const void* v, void* o, const osp_shape* shape, float softmax_scale,
                   void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (shape->text_len < 1)
    return set_error(OSP_ERR_INVALID_ARG, "cross-attention needs text_len >= 1 key/value tokens");
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return cross_attention_launch(q, k, v, o, *shape, softmax_scale, static_cast<cudaStream_t>(stream));
}

int osp_attn_spatial(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                     float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (shape->text_len != 0) return set_error(OSP_ERR_UNSUPPORTED, "spatial attention takes video tokens only (text_len 0)");
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if ((long long)shape->B * shape->T > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "too many frames");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  // [B][T*H*W][heads][d] is [B*T][H*W][heads][d]: one dense problem per frame
  const osp_shape frames{shape->B * shape->T, 0, 1, 1, shape->H * shape->W, shape->heads, shape->head_dim};
  return attention_launch(q, k, v, o, frames, 0, 1, softmax_scale, static_cast<cudaStream_t>(stream));
}

int osp_attn_temporal(const void* q, const void* k, const void* v, void* o, const osp_shape* shape, int32_t causal,
                      float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (shape->text_len != 0)
    return set_error(OSP_ERR_UNSUPPORTED, "temporal attention takes video tokens only (text_len 0)");
  if (causal != 0 && causal != 1) return set_error(OSP_ERR_INVALID_ARG, "causal must be 0 or 1 (got %d)", causal);
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->T <= 64) return temporal_attention_launch(q, k, v, o, *shape, causal, softmax_scale, st);
  // longer sets: the position's tokens t*H*W + pos are Single Skip set pos with k = H*W
  if (causal) return causal_temporal_attention_launch(q, k, v, o, *shape, softmax_scale, st);
  return attention_launch(q, k, v, o, *shape, OSP_SKIP_SINGLE + 1, shape->H * shape->W, softmax_scale, st);
}

int osp_attn_frame_causal(const void* q, const void* k, const void* v, void* o, const osp_shape* shape,
                          float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return frame_causal_attention_launch(q, k, v, o, *shape, softmax_scale, static_cast<cudaStream_t>(stream));
}

// Shared validation of the training entry points: dense (sparse_k == 1, text allowed) or
// Skiparse (sparse_k > 1, video tokens only).
static int check_train(const osp_shape* shape, int32_t sparse_k, int32_t mode, int* layout) {
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (sparse_k == 1) {
    *layout = 0;
    return OSP_OK;
  }
  if ((rc = check_skiparse(shape, sparse_k, mode, true))) return rc;
  if (mode == OSP_SKIP_GROUP && (sparse_k > 128 || (128 % sparse_k) != 0))
    return set_error(OSP_ERR_UNSUPPORTED, "fused Group Skip needs k to divide 128 (got k=%d)", sparse_k);
  *layout = mode + 1;
  return OSP_OK;
}

int osp_attn_forward_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                           int32_t sparse_k, int32_t mode, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int layout = 0;
  int rc = check_train(shape, sparse_k, mode, &layout);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  if (shape->text_len > 0 && layout != 0)
    return skiparse_text_attention_launch(q, k, v, o, *shape, sparse_k, mode, softmax_scale,
                                          static_cast<cudaStream_t>(stream), lse);
  return attention_forward_lse_launch(q, k, v, o, lse, *shape, layout, sparse_k, softmax_scale,
                                      static_cast<cudaStream_t>(stream));
}

int osp_attn_backward(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                      void* dq, void* dk, void* dv, const osp_shape* shape, int32_t sparse_k, int32_t mode,
                      float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int layout = 0;
  int rc = check_train(shape, sparse_k, mode, &layout);
  if (rc) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  if (shape->text_len > 0 && layout != 0)
    return skiparse_text_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, *shape, sparse_k, mode, softmax_scale,
                                         static_cast<cudaStream_t>(stream));
  return attention_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, *shape, layout, sparse_k, softmax_scale,
                                   static_cast<cudaStream_t>(stream));
}

int osp_attn_frame_causal_train(const void* q, const void* k, const void* v, void* o, float* lse,
                                const osp_shape* shape, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return attention_forward_lse_launch(q, k, v, o, lse, *shape, 0, 1, softmax_scale, static_cast<cudaStream_t>(stream),
                                      true);
}

int osp_attn_frame_causal_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                                   const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape,
                                   float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return attention_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, *shape, 0, 1, softmax_scale,
                                   static_cast<cudaStream_t>(stream), true);
}

// Factorized (2D + 1D) training: per-frame attention is dense attention over the frames
// [B*T][H*W]; the temporal set of spatial position pos is Single Skip set pos with k = H*W
// (slot t = frame t), causal through the block-causal mask with one-slot blocks.
static int check_factorized(const osp_shape* shape, const char* what) {
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if (shape->text_len != 0)
    return set_error(OSP_ERR_UNSUPPORTED, "%s attention takes video tokens only (text_len 0)", what);
  if ((long long)shape->B * shape->T > (1LL << 30) || (long long)shape->B * shape->H * shape->W > (1LL << 30))
    return set_error(OSP_ERR_UNSUPPORTED, "too many frames or positions");
  return OSP_OK;
}

static bool fwd_ptrs_ok(const void* q, const void* k, const void* v, const void* o, const void* lse) {
  if (!q || !k || !v || !o || !lse) {
    set_error(OSP_ERR_INVALID_ARG, "null pointer");
    return false;
  }
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse)) {
    set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    return false;
  }
  return true;
}

static bool bwd_ptrs_ok(const void* q, const void* k, const void* v, const void* o, const void* dout, const void* lse,
                        const void* dq, const void* dk, const void* dv) {
  if (!fwd_ptrs_ok(q, k, v, o, lse)) return false;
  if (!dout || !dq || !dk || !dv) {
    set_error(OSP_ERR_INVALID_ARG, "null pointer");
    return false;
  }
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) {
    set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    return false;
  }
  return true;
}

// T <= 64: the per-set temporal kernels for the training forward and the backward, unless
// OSP_TEMPORAL_BWD=0 selects the Skiparse kernels on one 128-row tile per set.  Read on every call.
static bool temporal_bwd_kernel() {
  const char* e = std::getenv("OSP_TEMPORAL_BWD");
  return e == nullptr || std::atoi(e) != 0;
}

static osp_shape frames_of(const osp_shape& s) {
  return osp_shape{s.B * s.T, 0, 1, 1, s.H * s.W, s.heads, s.head_dim};
}

int osp_attn_spatial_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                           float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_factorized(shape, "spatial");
  if (rc) return rc;
  if (!fwd_ptrs_ok(q, k, v, o, lse)) return OSP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return attention_forward_lse_launch(q, k, v, o, lse, frames_of(*shape), 0, 1, softmax_scale,
                                      static_cast<cudaStream_t>(stream));
}

int osp_attn_spatial_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                              const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape,
                              float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_factorized(shape, "spatial");
  if (rc) return rc;
  if (!bwd_ptrs_ok(q, k, v, o, dout, lse, dq, dk, dv)) return OSP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  return attention_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, frames_of(*shape), 0, 1, softmax_scale,
                                   static_cast<cudaStream_t>(stream));
}

int osp_attn_temporal_train(const void* q, const void* k, const void* v, void* o, float* lse, const osp_shape* shape,
                            int32_t causal, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_factorized(shape, "temporal");
  if (rc) return rc;
  if (causal != 0 && causal != 1) return set_error(OSP_ERR_INVALID_ARG, "causal must be 0 or 1 (got %d)", causal);
  if (!fwd_ptrs_ok(q, k, v, o, lse)) return OSP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  const int HW = shape->H * shape->W;
  if (shape->T <= 64 && temporal_bwd_kernel())
    return temporal_attention_launch(q, k, v, o, *shape, causal, softmax_scale, static_cast<cudaStream_t>(stream),
                                     lse);
  return attention_forward_lse_launch(q, k, v, o, lse, *shape, HW > 1 ? OSP_SKIP_SINGLE + 1 : 0, HW, softmax_scale,
                                      static_cast<cudaStream_t>(stream), causal != 0, 1);
}

int osp_attn_temporal_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                               const float* lse, void* dq, void* dk, void* dv, const osp_shape* shape, int32_t causal,
                               float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_factorized(shape, "temporal");
  if (rc) return rc;
  if (causal != 0 && causal != 1) return set_error(OSP_ERR_INVALID_ARG, "causal must be 0 or 1 (got %d)", causal);
  if (!bwd_ptrs_ok(q, k, v, o, dout, lse, dq, dk, dv)) return OSP_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  const int HW = shape->H * shape->W;
  if (shape->T <= 64 && temporal_bwd_kernel())
    return temporal_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, *shape, causal, softmax_scale,
                                    static_cast<cudaStream_t>(stream));
  return attention_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, *shape, HW > 1 ? OSP_SKIP_SINGLE + 1 : 0, HW,
                                   softmax_scale, static_cast<cudaStream_t>(stream), causal != 0, 1);
}

int osp_rope3d_packed(const void* q, const void* k, void* q_out, void* k_out, const osp_sample_grid* samples,
                      int32_t n_samples, int32_t heads, int32_t head_dim, const osp_rope* rope, void* stream) {
  g_last_error[0] = 0;
  if (!samples) return set_error(OSP_ERR_INVALID_ARG, "samples is NULL");
  if (n_samples < 1 || n_samples > OSP_MAX_SEGMENTS)
    return set_error(n_samples < 1 ? OSP_ERR_INVALID_ARG : OSP_ERR_UNSUPPORTED, "n_samples = %d not in [1, %d]",
                     n_samples, OSP_MAX_SEGMENTS);
  long long total = 0;
  for (int i = 0; i < n_samples; ++i) {
    const osp_sample_grid& g = samples[i];
    const osp_shape one{1, g.text_len, g.T, g.H, g.W, heads, head_dim};
    int rc = check_shape(&one, false);
    if (rc) {
      char msg[256];
      snprintf(msg, sizeof(msg), "%s", g_last_error);
      return set_error(rc, "sample %d: %s", i, msg);
    }
    total += (long long)g.text_len + (long long)g.T * g.H * g.W;
  }
  if (total > (1LL << 30)) return set_error(OSP_ERR_UNSUPPORTED, "packed batch of %lld rows is too large", total);
  int rc = check_rope(rope, head_dim);
  if (rc) return rc;
  if (!q || !k || !q_out || !k_out) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(q_out) || !aligned16(k_out))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return rope3d_packed_launch(q, k, q_out, k_out, samples, n_samples, heads, head_dim, *rope,
                              static_cast<cudaStream_t>(stream));
}

int osp_attn_packed(const void* q, const void* k, const void* v, void* o, const int32_t* q_bounds,
                    const int32_t* kv_bounds, int32_t n_seg, int32_t heads, int32_t head_dim, float softmax_scale,
                    void* stream) {
  g_last_error[0] = 0;
  if (n_seg < 1 || n_seg > OSP_MAX_SEGMENTS)
    return set_error(n_seg < 1 ? OSP_ERR_INVALID_ARG : OSP_ERR_UNSUPPORTED, "n_seg = %d not in [1, %d]", n_seg,
                     OSP_MAX_SEGMENTS);
  if (heads < 1) return set_error(OSP_ERR_INVALID_ARG, "heads = %d", heads);
  if (head_dim != 64 && head_dim != 96 && head_dim != 128)
    return set_error(OSP_ERR_UNSUPPORTED, "attention head_dim %d not in {64, 96, 128}", head_dim);
  int rc = check_bounds(q_bounds, n_seg, "q_bounds");
  if (rc) return rc;
  if (!kv_bounds) kv_bounds = q_bounds;
  if ((rc = check_bounds(kv_bounds, n_seg, "kv_bounds"))) return rc;
  for (int i = 0; i < n_seg; ++i)
    if (q_bounds[i + 1] > q_bounds[i] && kv_bounds[i + 1] == kv_bounds[i])
      return set_error(OSP_ERR_INVALID_ARG, "sample %d has %d query rows and no key rows", i,
                       q_bounds[i + 1] - q_bounds[i]);
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)head_dim);
  return packed_attention_launch(q, k, v, o, q_bounds, kv_bounds, n_seg, heads, head_dim, softmax_scale,
                                 static_cast<cudaStream_t>(stream));
}

static int check_packed_call(const int32_t* bounds, int32_t n_seg, int32_t heads, int32_t head_dim) {
  if (n_seg < 1 || n_seg > OSP_MAX_SEGMENTS)
    return set_error(n_seg < 1 ? OSP_ERR_INVALID_ARG : OSP_ERR_UNSUPPORTED, "n_seg = %d not in [1, %d]", n_seg,
                     OSP_MAX_SEGMENTS);
  if (heads < 1) return set_error(OSP_ERR_INVALID_ARG, "heads = %d", heads);
  if (head_dim != 64 && head_dim != 96 && head_dim != 128)
    return set_error(OSP_ERR_UNSUPPORTED, "attention head_dim %d not in {64, 96, 128}", head_dim);
  return check_bounds(bounds, n_seg, "bounds");
}

int osp_attn_packed_lse_rows(const int32_t* bounds, int32_t n_seg) {
  g_last_error[0] = 0;
  if (n_seg < 1 || n_seg > OSP_MAX_SEGMENTS) return -set_error(OSP_ERR_INVALID_ARG, "n_seg = %d", n_seg);
  const int rc = check_bounds(bounds, n_seg, "bounds");
  if (rc) return -rc;
  return packed_lse_rows(bounds, n_seg);
}

int osp_attn_packed_train(const void* q, const void* k, const void* v, void* o, float* lse, const int32_t* bounds,
                          int32_t n_seg, int32_t heads, int32_t head_dim, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_packed_call(bounds, n_seg, heads, head_dim);
  if (rc) return rc;
  if (!q || !k || !v || !o || !lse) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse))
    return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)head_dim);
  return packed_attention_launch(q, k, v, o, bounds, bounds, n_seg, heads, head_dim, softmax_scale,
                                 static_cast<cudaStream_t>(stream), lse);
}

int osp_attn_packed_backward(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, void* dq, void* dk, void* dv, const int32_t* bounds, int32_t n_seg,
                             int32_t heads, int32_t head_dim, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_packed_call(bounds, n_seg, heads, head_dim);
  if (rc) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return set_error(OSP_ERR_INVALID_ARG, "null pointer");
  for (const void* t : {q, k, v, o, dout, static_cast<const void*>(lse), static_cast<const void*>(dq),
                        static_cast<const void*>(dk), static_cast<const void*>(dv)})
    if (!aligned16(t)) return set_error(OSP_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)head_dim);
  return packed_backward_launch(q, k, v, o, dout, lse, dq, dk, dv, bounds, n_seg, heads, head_dim, softmax_scale,
                                static_cast<cudaStream_t>(stream));
}

int osp_skiparse_gather(const void* q, const void* k, const void* v, void* q_out, void* k_out, void* v_out,
                        const osp_shape* shape, int32_t sparse_k, int32_t mode, const osp_rope* rope, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, false);
  if (rc) return rc;
  if ((rc = check_skiparse(shape, sparse_k, mode))) return rc;
  if (rope && (rc = check_rope(rope, shape->head_dim))) return rc;
  if (!q || !q_out) return set_error(OSP_ERR_INVALID_ARG, "q and q_out must not be NULL");
  if ((!k) != (!k_out) || (!v) != (!v_out))
    return set_error(OSP_ERR_INVALID_ARG, "k/k_out and v/v_out must be both set or both NULL");
  const void* src[3];
  void* dst[3];
  int n = 0;
  src[n] = q; dst[n++] = q_out;
  if (k) { src[n] = k; dst[n++] = k_out; }
  if (v) { src[n] = v; dst[n++] = v_out; }
  for (int i = 0; i < n; ++i)
    if (!aligned16(src[i]) || !aligned16(dst[i]))
      return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  // RoPE applies to q and k only; with k omitted, v (if given) must not be rotated.
  if (rope && !k && v) {
    rc = skiparse_gather_launch(src, dst, 1, *shape, sparse_k, mode, rope, static_cast<cudaStream_t>(stream));
    if (rc) return rc;
    const void* s2[3] = {v, nullptr, nullptr};
    void* d2[3] = {v_out, nullptr, nullptr};
    return skiparse_gather_launch(s2, d2, 1, *shape, sparse_k, mode, nullptr, static_cast<cudaStream_t>(stream));
  }
  return skiparse_gather_launch(src, dst, n, *shape, sparse_k, mode, rope, static_cast<cudaStream_t>(stream));
}

int osp_skiparse_scatter(const void* o_perm, void* o, const osp_shape* shape, int32_t sparse_k, int32_t mode,
                         void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, false);
  if (rc) return rc;
  if ((rc = check_skiparse(shape, sparse_k, mode))) return rc;
  if (!o_perm || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(o_perm) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  return skiparse_scatter_launch(o_perm, o, *shape, sparse_k, mode, static_cast<cudaStream_t>(stream));
}

int osp_skiparse_attn(const void* q, const void* k, const void* v, void* o, const osp_shape* shape, int32_t sparse_k,
                      int32_t mode, float softmax_scale, void* stream) {
  g_last_error[0] = 0;
  int rc = check_shape(shape, true);
  if (rc) return rc;
  if ((rc = check_skiparse(shape, sparse_k, mode, true))) return rc;
  if (mode == OSP_SKIP_GROUP && (sparse_k > 128 || (128 % sparse_k) != 0))
    return set_error(OSP_ERR_UNSUPPORTED, "fused Group Skip needs k to divide 128 (got k=%d)", sparse_k);
  if (!q || !k || !v || !o) return set_error(OSP_ERR_INVALID_ARG, "null tensor pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return set_error(OSP_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
  if (!(softmax_scale > 0.f)) softmax_scale = 1.0f / std::sqrt((float)shape->head_dim);
  const int layout = (sparse_k == 1) ? 0 : (mode == OSP_SKIP_SINGLE ? 1 : 2);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (shape->text_len > 0 && layout != 0)
    return skiparse_text_attention_launch(q, k, v, o, *shape, sparse_k, mode, softmax_scale, st);
  return attention_launch(q, k, v, o, *shape, layout, sparse_k, softmax_scale, st);
}

int osp_skiparse_index_map(int32_t n_video, int32_t sparse_k, int32_t mode, int32_t* dev_out, void* stream) {
  g_last_error[0] = 0;
  if (n_video < 1) return set_error(OSP_ERR_INVALID_ARG, "n_video=%d < 1", n_video);
  if (!dev_out) return set_error(OSP_ERR_INVALID_ARG, "dev_out is NULL");
  osp_shape s{1, 0, 1, 1, n_video, 1, 8};
  int rc = check_skiparse(&s, sparse_k, mode);
  if (rc) return rc;
  return index_map_launch(n_video, sparse_k, mode, dev_out, static_cast<cudaStream_t>(stream));
}

int osp_check_status(void* stream) {
  g_last_error[0] = 0;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return set_error(OSP_ERR_CUDA, "stream synchronize failed: %s", cudaGetErrorString(e));
  // Both words of this device, where they exist: a word that was never created was never
  // written, and creating one here would allocate (which allocation-free callers cannot have).
  unsigned h = 0;
  for (unsigned* w : {device_status_word_if_present(), noalloc_status_word_if_present()}) {
    if (!w) continue;
    unsigned x = 0;
    if (cudaMemcpy(&x, w, sizeof(x), cudaMemcpyDeviceToHost) != cudaSuccess ||
        cudaMemset(w, 0, sizeof(unsigned)) != cudaSuccess)
      return set_error(OSP_ERR_CUDA, "status word read failed");
    h |= x;
  }
  if (h & kDevTimeout) return set_error(OSP_ERR_TIMEOUT, "a device-side bounded wait timed out");
  if (h & kDevBounds) return set_error(OSP_ERR_BOUNDS, "a device-side index check failed");
  return OSP_OK;
}

}  // extern "C"
