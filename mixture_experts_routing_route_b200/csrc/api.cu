// The extern "C" entry points of libmoe_b200.so: argument checks, workspace
// layout, and the stage launches on the caller's stream. Nothing here
// allocates device memory or synchronises, except moe_get_device_error.
#include "common.cuh"
#include <atomic>
#include <climits>
#include <cmath>

namespace moe {

namespace {
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t esize(moe_dtype_t dt) { return dt == MOE_BF16 ? 2 : 4; }

moe_status_t check_dims(moe_dtype_t dt, int T, int d, int E, int k) {
  if (dt != MOE_BF16 && dt != MOE_F32) return MOE_ERR_INVALID;
  if (T < 0 || d <= 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID;
  if (static_cast<long long>(T) * k >= INT_MAX) return MOE_ERR_INVALID;
  if (dt == MOE_BF16 && d % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_F32 && d % 4 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_ffn(moe_dtype_t dt, int F) {
  if (F <= 0) return MOE_ERR_INVALID;
  if (dt == MOE_BF16 && F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (dt == MOE_F32 && F % 4 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_CHECK(expr)                      \
  do {                                       \
    const moe_status_t st_ = (expr);         \
    if (st_ != MOE_OK) return st_;           \
  } while (0)

#define MOE_NEED(p)                                  \
  do {                                               \
    if ((p) == nullptr) return MOE_ERR_NULL;         \
    if (!aligned16(p)) return MOE_ERR_ALIGN;         \
  } while (0)

#define MOE_OPT(p)                                   \
  do {                                               \
    if ((p) != nullptr && !aligned16(p)) return MOE_ERR_ALIGN; \
  } while (0)

// Bump allocator over a workspace, 256-byte aligned pieces.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += align_up(bytes);
    return p;
  }
};

struct FwdLayout {
  Control* ctl;
  void* partials;
  float* logits_scratch;
  int32_t* idx;
  float* w;
  float* aux;
  float* z;  // z-loss (MOE_LAYER_Z_LOSS)
  int32_t *counts, *bins, *kept, *seg;
  int32_t *sorted_slot, *slot_to_row, *row_slot;
  uint8_t* drop;
  int32_t* rank;
  void *x_perm, *h, *y_perm;
  void *x_dev, *out_dev;  // host-buffer variant only
  int64_t cap, rows_max;
  size_t bytes;
};

bool binned(const moe_layer_t* L) { return (L->flags & MOE_LAYER_BINNED) != 0; }

bool gather_in_gemm(const moe_layer_t* L) {
  return L->dtype == MOE_BF16 && (L->flags & MOE_LAYER_GATHER_IN_GEMM) != 0;
}

bool combine_in_gemm(const moe_layer_t* L) {
  return L->dtype == MOE_BF16 && L->k == 1 && (L->flags & MOE_LAYER_COMBINE_IN_GEMM) != 0;
}

FwdLayout fwd_layout(const moe_layer_t* L, int T, void* ws, bool host_io) {
  FwdLayout f{};
  Carver c(ws);
  const size_t S = static_cast<size_t>(T) * L->k;
  const size_t es = esize(L->dtype);
  f.cap = moe_capacity(L->capacity_factor, T, L->k, L->E);
  f.rows_max = binned(L) ? moe_rows_max_binned(T, L->k, L->E, f.cap)
                         : moe_rows_max(T, L->k, L->E, f.cap);
  const size_t R = static_cast<size_t>(f.rows_max);
  f.ctl = static_cast<Control*>(c.take(sizeof(Control)));
  f.partials = c.take(route_partials_bytes(T, L->E));
  f.logits_scratch = static_cast<float*>(c.take(route_logits_scratch_bytes(T, L->d, L->E)));
  f.idx = static_cast<int32_t*>(c.take(S * 4));
  f.w = static_cast<float*>(c.take(S * 4));
  f.aux = static_cast<float*>(c.take(4));
  f.z = static_cast<float*>(c.take(4));
  f.counts = static_cast<int32_t*>(c.take(L->E * 4));
  f.bins = static_cast<int32_t*>(c.take(L->E * 4));
  f.kept = static_cast<int32_t*>(c.take(L->E * 4));
  f.seg = static_cast<int32_t*>(c.take((L->E + 1) * 4));
  f.sorted_slot = static_cast<int32_t*>(c.take(S * 4));
  f.slot_to_row = static_cast<int32_t*>(c.take(S * 4));
  f.row_slot = static_cast<int32_t*>(c.take(R * 4));
  f.drop = static_cast<uint8_t*>(c.take(S));
  f.rank = static_cast<int32_t*>(c.take(permute_scratch_bytes(T, L->k, L->E)));
  // With MOE_LAYER_GATHER_IN_GEMM the up projection gathers the token rows
  // itself and there is no x_perm.
  f.x_perm = gather_in_gemm(L) ? nullptr : c.take(R * L->d * es);
  f.h = c.take(R * L->F * es);
  // With MOE_LAYER_COMBINE_IN_GEMM the down projection writes out itself.
  f.y_perm = combine_in_gemm(L) ? nullptr : c.take(R * L->d * es);
  if (host_io) {
    f.x_dev = c.take(static_cast<size_t>(T) * L->d * es);
    f.out_dev = c.take(static_cast<size_t>(T) * L->d * es);
  }
  f.bytes = c.off;
  return f;
}

moe_status_t check_layer(const moe_layer_t* L, int T) {
  if (L == nullptr) return MOE_ERR_NULL;
  MOE_CHECK(check_dims(L->dtype, T, L->d, L->E, L->k));
  MOE_CHECK(check_ffn(L->dtype, L->F));
  if (L->act != MOE_ACT_GELU && L->act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID;
  if (!std::isfinite(L->capacity_factor)) return MOE_ERR_INVALID;
  if (!(L->router_temperature >= 0.0f) || !std::isfinite(L->router_temperature)) return MOE_ERR_INVALID;
  if ((L->flags & ~(MOE_LAYER_GATHER_IN_GEMM | MOE_LAYER_BINNED | MOE_LAYER_Z_LOSS |
                    MOE_LAYER_COMBINE_IN_GEMM)) != 0)
    return MOE_ERR_INVALID;
  MOE_OPT(L->x_router);
  MOE_OPT(L->logit_noise);
  if ((L->flags & MOE_LAYER_GATHER_IN_GEMM) && L->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  if ((L->flags & MOE_LAYER_COMBINE_IN_GEMM) && (L->dtype != MOE_BF16 || L->k != 1))
    return MOE_ERR_UNSUPPORTED;
  MOE_NEED(L->w_router);
  MOE_NEED(L->w1);
  MOE_NEED(L->w2);
  if (L->act == MOE_ACT_SWIGLU) MOE_NEED(L->w3);
  MOE_OPT(L->router_bias);
  return MOE_OK;
}

moe_status_t run_forward(const moe_layer_t* L, const void* x, int T, void* out, float* aux_user,
                         const FwdLayout& f, cudaStream_t s, const moe_event_t* ev) {
  auto rec = [&](int i) {
    if (ev != nullptr && ev[i] != nullptr) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s);
  };
  const size_t es = esize(L->dtype);
  rec(0);
  // the router may read its own input (a jittered x) and add logit noise; the
  // last step of its load-balance loss may run in the multi-CTA permute
  // kernel's tail instead of a launch of its own (launch_route decides)
  AuxJob aux_job{};
  AuxJob* defer = permute_uses_grid(T, L->k, L->E) ? &aux_job : nullptr;
  MOE_CHECK(from_cuda(launch_route(L->x_router != nullptr ? L->x_router : x, L->w_router,
                                   L->router_bias, L->logit_noise, L->dtype, T, L->d, L->E, L->k,
                                   f.idx, f.w, f.aux, (L->flags & MOE_LAYER_Z_LOSS) ? f.z : nullptr,
                                   nullptr, nullptr, f.logits_scratch, f.partials, f.ctl, s,
                                   L->router_temperature > 0.0f ? L->router_temperature : 1.0f,
                                   defer)));
  rec(1);
  MOE_CHECK(from_cuda(launch_permute(f.idx, T, L->k, L->E, f.cap, f.counts, f.bins, f.sorted_slot,
                                     f.slot_to_row, f.row_slot, f.drop, f.kept, f.seg, f.rank,
                                     f.ctl, s, binned(L),
                                     defer != nullptr && defer->pending ? defer : nullptr)));
  rec(2);
  const bool cig = combine_in_gemm(L);
  // the gather kernel also zeroes the output rows of fully dropped tokens
  // when the down projection writes out
  if (!gather_in_gemm(L) || cig)
    MOE_CHECK(from_cuda(launch_gather(x, es, T, L->d, L->k, f.row_slot, f.seg, L->E, f.rows_max,
                                      f.x_perm, f.ctl, s, binned(L), cig ? f.slot_to_row : nullptr,
                                      cig ? out : nullptr)));
  rec(3);
  cudaEvent_t after_up = (ev != nullptr) ? reinterpret_cast<cudaEvent_t>(ev[4]) : nullptr;
  if (L->dtype == MOE_BF16) {
    const bool g = gather_in_gemm(L);
    const CombineOut co{f.row_slot, f.w, out, T};
    MOE_CHECK(from_cuda(launch_ffn_bf16(g ? x : f.x_perm, g ? T : f.rows_max,
                                        g ? f.row_slot : nullptr, L->k, L->w1, L->w3, L->w2,
                                        L->act, f.rows_max, L->d, L->F, L->E, f.seg,
                                        binned(L) ? f.kept : nullptr, f.h, f.y_perm, f.ctl, s,
                                        after_up, cig ? &co : nullptr,
                                        static_cast<int64_t>(T) * L->k)));
  } else {
    MOE_CHECK(from_cuda(launch_ffn_f32(static_cast<const float*>(f.x_perm),
                                       static_cast<const float*>(L->w1),
                                       static_cast<const float*>(L->w3),
                                       static_cast<const float*>(L->w2), L->act, f.rows_max, L->d,
                                       L->F, L->E, f.seg, static_cast<float*>(f.h),
                                       static_cast<float*>(f.y_perm), f.ctl, s, after_up)));
  }
  rec(5);
  if (!cig)
    MOE_CHECK(from_cuda(launch_combine(f.y_perm, f.w, f.slot_to_row, es, T, L->d, L->k, f.rows_max,
                                       out, f.ctl, s)));
  rec(6);
  if (aux_user != nullptr && aux_user != f.aux)
    MOE_CHECK(from_cuda(cudaMemcpyAsync(aux_user, f.aux, 4, cudaMemcpyDeviceToDevice, s)));
  return MOE_OK;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(moe_status_t st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_NULL: return "a required pointer is NULL";
    case MOE_ERR_INVALID: return "a size or parameter is out of range";
    case MOE_ERR_UNSUPPORTED: return "shape outside this build's limits";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_ALIGN: return "pointer not 16-byte aligned";
    case MOE_ERR_CUDA: return "CUDA call or kernel launch failed";
    case MOE_ERR_DEVICE: return "device error word is set";
  }
  return "unknown status";
}

uint64_t moe_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

moe_status_t moe_workspace_init(void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  return from_cuda(cudaMemsetAsync(ws, 0, sizeof(Control), reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_workspace_set_wait_limit(void* ws, size_t ws_bytes, uint32_t limit_us,
                                          moe_stream_t stream) {
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  return from_cuda(launch_set_wait_limit(static_cast<Control*>(ws), limit_us,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_get_device_error(void* ws, moe_stream_t stream, uint32_t* host_bits, int clear) {
  MOE_NEED(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaMemcpyAsync(&v, &static_cast<Control*>(ws)->err, 4, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (clear && cudaMemsetAsync(&static_cast<Control*>(ws)->err, 0, 4, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (host_bits) *host_bits = v;
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

int64_t moe_capacity(double cf, int T, int k, int E) {
  if (!(cf > 0.0) || E <= 0) return -1;
  const double c = cf * (static_cast<double>(k) * static_cast<double>(T) / static_cast<double>(E));
  return static_cast<int64_t>(c);  // truncation toward zero, as int() does
}

int64_t moe_rows_max_binned(int T, int k, int E, int64_t capacity) {
  const int64_t S = static_cast<int64_t>(T) * k;
  return static_cast<int64_t>(E) * (capacity < 0 ? S : capacity);
}

int64_t moe_rows_max(int T, int k, int E, int64_t capacity) {
  const int64_t S = static_cast<int64_t>(T) * k;
  if (capacity < 0) return S;
  const int64_t ec = static_cast<int64_t>(E) * capacity;
  return ec < S ? ec : S;
}

size_t moe_route_workspace_size(int T, int d, int E) {
  if (T < 0 || E < 1) return 0;
  return align_up(sizeof(Control)) + route_partials_bytes(T, E) + route_logits_scratch_bytes(T, d, E);
}

static moe_status_t route_impl(const void* x, const void* w_router, const float* bias,
                               const float* logit_noise, float temperature, moe_dtype_t dtype,
                               int T, int d, int E, int k, int32_t* topk_idx, float* topk_w,
                               float* aux_loss, float* z_loss, float* logits, float* probs,
                               void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK(check_dims(dtype, T, d, E, k));
  if (!(temperature > 0.0f) || !std::isfinite(temperature)) return MOE_ERR_INVALID;
  MOE_NEED(x);
  MOE_NEED(w_router);
  MOE_NEED(topk_idx);
  MOE_NEED(topk_w);
  MOE_NEED(aux_loss);
  MOE_NEED(ws);
  MOE_OPT(bias);
  MOE_OPT(logit_noise);
  MOE_OPT(z_loss);
  MOE_OPT(logits);
  MOE_OPT(probs);
  if (ws_bytes < moe_route_workspace_size(T, d, E)) return MOE_ERR_WORKSPACE;
  Carver c(ws);
  Control* ctl = static_cast<Control*>(c.take(sizeof(Control)));
  void* partials = c.take(route_partials_bytes(T, E));
  float* scratch = static_cast<float*>(c.take(route_logits_scratch_bytes(T, d, E)));
  return from_cuda(launch_route(x, w_router, bias, logit_noise, dtype, T, d, E, k, topk_idx, topk_w,
                                aux_loss, z_loss, logits, probs, scratch, partials, ctl,
                                reinterpret_cast<cudaStream_t>(stream), temperature));
}

moe_status_t moe_route(const void* x, const void* w_router, const float* bias, moe_dtype_t dtype,
                       int T, int d, int E, int k, int32_t* topk_idx, float* topk_w, float* aux_loss,
                       float* logits, float* probs, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return route_impl(x, w_router, bias, nullptr, 1.0f, dtype, T, d, E, k, topk_idx, topk_w, aux_loss,
                    nullptr, logits, probs, ws, ws_bytes, stream);
}

moe_status_t moe_route_train(const void* x, const void* w_router, const float* bias,
                             const float* logit_noise, float temperature, moe_dtype_t dtype, int T,
                             int d, int E, int k, int32_t* topk_idx, float* topk_w,
                             float* aux_loss, float* z_loss, float* logits, float* probs, void* ws,
                             size_t ws_bytes, moe_stream_t stream) {
  return route_impl(x, w_router, bias, logit_noise, temperature, dtype, T, d, E, k, topk_idx, topk_w,
                    aux_loss, z_loss, logits, probs, ws, ws_bytes, stream);
}

size_t moe_route_backward_workspace_size(int T, int d, int E) {
  if (T < 0 || d < 1 || E < 1) return 0;
  return align_up(sizeof(Control)) + route_backward_scratch_bytes(T, d, E);
}

moe_status_t moe_route_backward(const void* x, const void* w_router, moe_dtype_t dtype, int T,
                                int d, int E, int k, const float* probs, const float* logits,
                                const int32_t* topk_idx, const float* topk_w,
                                const float* d_topk_w, float d_aux, float d_z, float temperature,
                                float* d_logits, void* dx, float* d_wg, void* ws, size_t ws_bytes,
                                moe_stream_t stream) {
  MOE_CHECK(check_dims(dtype, T, d, E, k));
  if (d % 4 != 0) return MOE_ERR_UNSUPPORTED;  // 4 columns per vector access
  if (!(temperature > 0.0f) || !std::isfinite(temperature) || !std::isfinite(d_aux) ||
      !std::isfinite(d_z))
    return MOE_ERR_INVALID;
  MOE_NEED(ws);
  MOE_OPT(logits);
  MOE_OPT(d_topk_w);
  MOE_OPT(d_logits);
  MOE_OPT(dx);
  MOE_OPT(d_wg);
  if (T > 0) {
    MOE_NEED(probs);
    MOE_NEED(topk_idx);
    if (d_topk_w != nullptr) MOE_NEED(topk_w);
    if (d_z != 0.0f) MOE_NEED(logits);
    if (dx != nullptr || d_wg != nullptr) MOE_NEED(w_router);
    if (d_wg != nullptr) MOE_NEED(x);
  }
  if (ws_bytes < moe_route_backward_workspace_size(T, d, E)) return MOE_ERR_WORKSPACE;
  Carver c(ws);
  Control* ctl = static_cast<Control*>(c.take(sizeof(Control)));
  void* scratch = c.take(route_backward_scratch_bytes(T, d, E));
  return from_cuda(launch_route_backward(x, w_router, dtype, T, d, E, k, probs, logits, topk_idx,
                                         topk_w, d_topk_w, d_aux, d_z, temperature, d_logits, dx,
                                         d_wg, scratch, ctl, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_router_jitter(const void* x, moe_dtype_t dtype, int T, int d, float eps,
                               uint64_t seed, void* x_out, moe_stream_t stream) {
  if (dtype != MOE_BF16 && dtype != MOE_F32) return MOE_ERR_INVALID;
  if (T < 0 || d <= 0 || !(eps >= 0.0f && eps < 1.0f)) return MOE_ERR_INVALID;
  if (T > 0) {
    MOE_NEED(x);
    MOE_NEED(x_out);
  }
  return from_cuda(launch_jitter(x, dtype, static_cast<long long>(T) * d, eps, seed, x_out,
                                 reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_router_noise(int T, int E, float std_dev, uint64_t seed, float* noise_out,
                              moe_stream_t stream) {
  if (T < 0 || E < 1 || !(std_dev >= 0.0f) || !std::isfinite(std_dev)) return MOE_ERR_INVALID;
  if (T > 0) MOE_NEED(noise_out);
  return from_cuda(launch_logit_noise(static_cast<long long>(T) * E, std_dev, seed, noise_out,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_permute_workspace_size(int T, int k, int E) {
  if (T < 0 || k < 1) return 0;
  return align_up(sizeof(Control)) + permute_scratch_bytes(T, k, E);
}

static moe_status_t permute_impl(const int32_t* topk_idx, int T, int k, int E, int64_t capacity,
                                 int32_t* counts, int32_t* bins, int32_t* sorted_slot,
                                 int32_t* slot_to_row, int32_t* row_slot, uint8_t* drop_mask,
                                 int32_t* kept_counts, int32_t* seg_offsets, void* ws,
                                 size_t ws_bytes, moe_stream_t stream, bool bin) {
  if (T < 0 || E < 1 || E > 256 || k < 1 || k > 8 || k > E) return MOE_ERR_INVALID;
  if (static_cast<long long>(T) * k >= INT_MAX) return MOE_ERR_INVALID;
  const int64_t rows = bin ? moe_rows_max_binned(T, k, E, capacity) : moe_rows_max(T, k, E, capacity);
  if (rows >= INT_MAX) return MOE_ERR_INVALID;
  if (T > 0) {
    MOE_NEED(topk_idx);
    MOE_NEED(sorted_slot);
    MOE_NEED(slot_to_row);
    MOE_NEED(drop_mask);
    if (rows > 0) MOE_NEED(row_slot);
  }
  MOE_NEED(counts);
  MOE_NEED(bins);
  MOE_NEED(kept_counts);
  MOE_NEED(seg_offsets);
  MOE_NEED(ws);
  if (ws_bytes < moe_permute_workspace_size(T, k, E)) return MOE_ERR_WORKSPACE;
  Carver c(ws);
  Control* ctl = static_cast<Control*>(c.take(sizeof(Control)));
  int32_t* rank = static_cast<int32_t*>(c.take(permute_scratch_bytes(T, k, E)));
  return from_cuda(launch_permute(topk_idx, T, k, E, capacity, counts, bins, sorted_slot,
                                  slot_to_row, row_slot, drop_mask, kept_counts, seg_offsets, rank,
                                  ctl, reinterpret_cast<cudaStream_t>(stream), bin));
}

moe_status_t moe_permute(const int32_t* topk_idx, int T, int k, int E, int64_t capacity,
                         int32_t* counts, int32_t* bins, int32_t* sorted_slot, int32_t* slot_to_row,
                         int32_t* row_slot, uint8_t* drop_mask, int32_t* kept_counts,
                         int32_t* seg_offsets, void* ws, size_t ws_bytes, moe_stream_t stream) {
  return permute_impl(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row, row_slot,
                      drop_mask, kept_counts, seg_offsets, ws, ws_bytes, stream, false);
}

moe_status_t moe_permute_binned(const int32_t* topk_idx, int T, int k, int E, int64_t capacity,
                                int32_t* counts, int32_t* bins, int32_t* sorted_slot,
                                int32_t* slot_to_row, int32_t* row_slot, uint8_t* drop_mask,
                                int32_t* kept_counts, int32_t* seg_offsets, void* ws,
                                size_t ws_bytes, moe_stream_t stream) {
  return permute_impl(topk_idx, T, k, E, capacity, counts, bins, sorted_slot, slot_to_row, row_slot,
                      drop_mask, kept_counts, seg_offsets, ws, ws_bytes, stream, true);
}

moe_status_t moe_gather(const void* x, moe_dtype_t dtype, int T, int d, int k,
                        const int32_t* row_slot, const int32_t* seg_offsets, int E, int64_t rows_max,
                        void* x_perm, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK(check_dims(dtype, T, d, E, k));
  if (rows_max < 0 || rows_max > static_cast<int64_t>(T) * k) return MOE_ERR_INVALID;
  MOE_NEED(seg_offsets);
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  if (rows_max > 0 && T > 0) {
    MOE_NEED(x);
    MOE_NEED(row_slot);
    MOE_NEED(x_perm);
  }
  return from_cuda(launch_gather(x, esize(dtype), T, d, k, row_slot, seg_offsets, E, rows_max,
                                 x_perm, static_cast<Control*>(ws),
                                 reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_expert_ffn(const void* x_perm, const void* w1, const void* w3, const void* w2,
                            moe_dtype_t dtype, moe_act_t act, int64_t rows_max, int d, int F, int E,
                            const int32_t* seg_offsets, void* h, void* y_perm, void* ws,
                            size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK(check_dims(dtype, 0, d, E, 1));
  MOE_CHECK(check_ffn(dtype, F));
  if (act != MOE_ACT_GELU && act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID;
  if (rows_max < 0 || rows_max >= INT_MAX) return MOE_ERR_INVALID;
  MOE_NEED(w1);
  MOE_NEED(w2);
  if (act == MOE_ACT_SWIGLU) MOE_NEED(w3);
  MOE_NEED(seg_offsets);
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  if (rows_max > 0) {
    MOE_NEED(x_perm);
    MOE_NEED(h);
    MOE_NEED(y_perm);
  }
  Control* ctl = static_cast<Control*>(ws);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == MOE_BF16)
    return from_cuda(launch_ffn_bf16(x_perm, rows_max, nullptr, 1, w1, w3, w2, act, rows_max, d, F,
                                     E, seg_offsets, nullptr, h, y_perm, ctl, s, nullptr));
  return from_cuda(launch_ffn_f32(static_cast<const float*>(x_perm), static_cast<const float*>(w1),
                                  static_cast<const float*>(w3), static_cast<const float*>(w2), act,
                                  rows_max, d, F, E, seg_offsets, static_cast<float*>(h),
                                  static_cast<float*>(y_perm), ctl, s, nullptr));
}

moe_status_t moe_combine(const void* y_perm, const float* topk_w, const int32_t* slot_to_row,
                         moe_dtype_t dtype, int T, int d, int k, int64_t rows_max, void* out, void* ws,
                         size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK(check_dims(dtype, T, d, k, k));
  if (rows_max < 0) return MOE_ERR_INVALID;
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  if (T > 0) {
    MOE_NEED(topk_w);
    MOE_NEED(slot_to_row);
    MOE_NEED(out);
    if (rows_max > 0) MOE_NEED(y_perm);
  }
  return from_cuda(launch_combine(y_perm, topk_w, slot_to_row, esize(dtype), T, d, k, rows_max, out,
                                  static_cast<Control*>(ws), reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_send_plan(const int32_t* kept_counts, const int32_t* seg_offsets, int E,
                              int world, int32_t* send_rows, int32_t* send_offsets, void* ws,
                              size_t ws_bytes, moe_stream_t stream) {
  if (E < 1 || E > 256 || world < 1 || E % world != 0) return MOE_ERR_INVALID;
  MOE_NEED(kept_counts);
  MOE_NEED(seg_offsets);
  MOE_NEED(send_rows);
  MOE_NEED(send_offsets);
  MOE_NEED(ws);
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  return from_cuda(launch_ep_send_plan(kept_counts, seg_offsets, world, E / world, send_rows,
                                       send_offsets, static_cast<Control*>(ws),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

moe_status_t moe_ep_recv_plan(const int32_t* recv_counts, int world, int experts_per_rank,
                              int64_t rows_cap, int32_t* recv_rows, int32_t* recv_offsets,
                              int32_t* local_seg, int32_t* local_to_recv, int32_t* recv_to_local,
                              void* ws, size_t ws_bytes, moe_stream_t stream) {
  if (world < 1 || experts_per_rank < 1 || static_cast<long long>(world) * experts_per_rank > 256)
    return MOE_ERR_INVALID;
  if (rows_cap < 0 || rows_cap >= INT_MAX) return MOE_ERR_INVALID;
  MOE_NEED(recv_counts);
  MOE_NEED(recv_rows);
  MOE_NEED(recv_offsets);
  MOE_NEED(local_seg);
  MOE_NEED(ws);
  if (rows_cap > 0) {
    MOE_NEED(local_to_recv);
    MOE_NEED(recv_to_local);
  }
  if (ws_bytes < sizeof(Control)) return MOE_ERR_WORKSPACE;
  return from_cuda(launch_ep_recv_plan(recv_counts, world, experts_per_rank, rows_cap, recv_rows,
                                       recv_offsets, local_seg, local_to_recv, recv_to_local,
                                       static_cast<Control*>(ws),
                                       reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_forward_workspace_size(const moe_layer_t* layer, int T) {
  if (layer == nullptr || T < 0) return 0;
  return fwd_layout(layer, T, nullptr, false).bytes;
}

size_t moe_forward_host_workspace_size(const moe_layer_t* layer, int T) {
  if (layer == nullptr || T < 0) return 0;
  return fwd_layout(layer, T, nullptr, true).bytes;
}

moe_status_t moe_forward_views(const moe_layer_t* layer, int T, void* ws, size_t ws_bytes,
                               moe_views_t* v) {
  MOE_CHECK(check_layer(layer, T));
  MOE_NEED(ws);
  if (v == nullptr) return MOE_ERR_NULL;
  const FwdLayout f = fwd_layout(layer, T, ws, false);
  if (ws_bytes < f.bytes) return MOE_ERR_WORKSPACE;
  v->topk_idx = f.idx;
  v->topk_w = f.w;
  v->aux_loss = f.aux;
  v->z_loss = f.z;
  v->counts = f.counts;
  v->bins = f.bins;
  v->kept_counts = f.kept;
  v->seg_offsets = f.seg;
  v->sorted_slot = f.sorted_slot;
  v->slot_to_row = f.slot_to_row;
  v->row_slot = f.row_slot;
  v->drop_mask = f.drop;
  v->x_perm = f.x_perm;
  v->h = f.h;
  v->y_perm = f.y_perm;
  v->rows_max = f.rows_max;
  v->capacity = f.cap;
  return MOE_OK;
}

moe_status_t moe_forward(const moe_layer_t* layer, const void* x, int T, void* out, float* aux_loss,
                         void* ws, size_t ws_bytes, moe_stream_t stream, const moe_event_t* events) {
  MOE_CHECK(check_layer(layer, T));
  MOE_NEED(ws);
  MOE_OPT(aux_loss);
  if (T > 0) {
    MOE_NEED(x);
    MOE_NEED(out);
  }
  const FwdLayout f = fwd_layout(layer, T, ws, false);
  if (ws_bytes < f.bytes) return MOE_ERR_WORKSPACE;
  return run_forward(layer, x, T, out, aux_loss, f, reinterpret_cast<cudaStream_t>(stream), events);
}

moe_status_t moe_forward_host(const moe_layer_t* layer, const void* x_host, int T, void* out_host,
                              float* aux_host, void* ws, size_t ws_bytes, moe_stream_t stream) {
  MOE_CHECK(check_layer(layer, T));
  MOE_NEED(ws);
  if (T > 0 && (x_host == nullptr || out_host == nullptr)) return MOE_ERR_NULL;
  const FwdLayout f = fwd_layout(layer, T, ws, true);
  if (ws_bytes < f.bytes) return MOE_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t bytes = static_cast<size_t>(T) * layer->d * esize(layer->dtype);
  if (bytes) MOE_CHECK(from_cuda(cudaMemcpyAsync(f.x_dev, x_host, bytes, cudaMemcpyHostToDevice, s)));
  MOE_CHECK(run_forward(layer, f.x_dev, T, f.out_dev, nullptr, f, s, nullptr));
  if (bytes) MOE_CHECK(from_cuda(cudaMemcpyAsync(out_host, f.out_dev, bytes, cudaMemcpyDeviceToHost, s)));
  if (aux_host) MOE_CHECK(from_cuda(cudaMemcpyAsync(aux_host, f.aux, 4, cudaMemcpyDeviceToHost, s)));
  return MOE_OK;
}

}  // extern "C"
