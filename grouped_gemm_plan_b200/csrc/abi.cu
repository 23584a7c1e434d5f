// abi.cu -- the extern "C" entry points of libmoe.so (declared in include/moe.h).
//
// Host-side work only: argument validation (before anything is launched),
// workspace carving, and kernel launches on the caller's stream.  Every step of
// the layer itself runs in the kernels of plan.cu, permute.cu and
// grouped_gemm.cu; there is no host or CPU fallback.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "common.cuh"

namespace moe {
cudaError_t launch_plan(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                        int32_t* status, int32_t* scratch, int num_sms, cudaStream_t stream);
cudaError_t launch_dispatch(const void* x, const int32_t* perm, int64_t M, int64_t H, int32_t topk,
                            void* xp, int32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_dispatch_tokens(const void* x, const int32_t* inv, int64_t M, int64_t H,
                                   int32_t topk, void* xp, int32_t* status, int num_sms,
                                   cudaStream_t stream);
cudaError_t launch_combine(const void* y, bool y_f32, const int32_t* inv, const float* w,
                           int64_t M, int64_t H, int32_t topk, void* out, int32_t* status,
                           int num_sms, cudaStream_t stream);
int launch_grouped_gemm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                        int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                        const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                        int num_sms, cudaStream_t stream);
cudaError_t launch_combine_add(const void* y, bool y_f32, const int32_t* inv, const float* w,
                               const void* add, float alpha, float beta, int64_t M, int64_t H,
                               int32_t topk, void* out, int32_t* status, int num_sms,
                               cudaStream_t stream);
size_t layer_sync_bytes(int64_t M, int64_t R, int32_t E);
cudaError_t launch_quantize_rows(const void* A, int64_t R, int64_t K, void* q, float* scale,
                                 int num_sms, cudaStream_t stream);
cudaError_t launch_quantize_cols(const void* W, int32_t E, int64_t K, int64_t N, void* qT,
                                 float* scale, cudaStream_t stream);
int launch_grouped_gemm_e4m3(const void* Aq, const float* a_scale, const void* BqT,
                             const float* b_scale, const int32_t* offsets, int32_t E, int64_t R,
                             int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                             float* C, int32_t* status, uint64_t timeout_ns, int num_sms,
                             cudaStream_t stream);
int launch_moe_layer(const void* x, const void* W1, const void* W2, const int32_t* perm,
                     const float* w_sorted, const int32_t* offsets, void* xp, void* h, void* yk,
                     void* out, int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk,
                     int32_t n_c, int32_t* status, void* sync_area, uint64_t timeout_ns,
                     int32_t withhold_mtile, int num_sms, cudaStream_t stream);
int32_t profiled_n_c(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk);
int launch_grouped_gemm_swiglu_mx(const void* A, const void* B, const int32_t* offsets, int32_t E,
                                  int64_t R, int64_t K, int64_t N2, uint8_t* q, uint8_t* sf,
                                  bool sf_row_major, int32_t kg_pad, int32_t* status,
                                  uint64_t timeout_ns, int num_sms, cudaStream_t stream);
int32_t mx_kg_pad(int64_t K);
size_t mx_sfa_bytes(int64_t R, int32_t E, int64_t K);
size_t mx_sfb_bytes(int32_t E, int64_t N, int64_t K);
cudaError_t launch_quantize_weights_mx(const void* W, int32_t E, int64_t K, int64_t N, void* BqT,
                                       uint8_t* sf, int num_sms, cudaStream_t stream);
cudaError_t launch_quantize_rows_mx(const void* A, int64_t R, int64_t K, void* Aq, uint8_t* sf,
                                    int num_sms, cudaStream_t stream);
cudaError_t launch_pack_sfa(const uint8_t* sf, const int32_t* offsets, int32_t E, int64_t R,
                            int64_t K, uint8_t* groups, int32_t* status, int num_sms,
                            cudaStream_t stream);
cudaError_t launch_pack_sfb(const uint8_t* sf, int32_t E, int64_t N, int64_t K, uint8_t* groups,
                            int num_sms, cudaStream_t stream);
int launch_grouped_gemm_mx(const void* Aq, const uint8_t* sfa_groups, const void* BqT,
                           const uint8_t* sfb_groups, const int32_t* offsets, int32_t E, int64_t R,
                           int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                           float* C, int32_t* status, uint64_t timeout_ns, int num_sms,
                           cudaStream_t stream);
cudaError_t launch_route(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* ids,
                         float* w, int num_sms, cudaStream_t stream);
cudaError_t launch_route_plan(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* ids,
                              float* w, int32_t* counts, int32_t* offsets, int32_t* perm,
                              int32_t* inv, float* w_sorted, int32_t* status, int32_t* scratch,
                              int num_sms, cudaStream_t stream);
}  // namespace moe

namespace {

thread_local std::string g_last_error;
uint64_t g_timeout_ns = 2000000000ull;
int32_t g_withhold_mtile = -1;  // fault injection for tests (moe_set_fault_injection)
thread_local cudaEvent_t g_stage_events[6];  // moe_set_stage_events
thread_local bool g_stage_events_on = false;

// Records stage event i of moe_ffn_fused when stage timing is on.
void stage_mark(int i, cudaStream_t s) {
  if (g_stage_events_on) cudaEventRecord(g_stage_events[i], s);
}

constexpr size_t kCtrlBytes = 256;
constexpr int64_t kMaxRows = (int64_t(1) << 31) - 1;

moe_status fail(moe_status st, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
moe_status fail(moe_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

moe_status cuda_fail(cudaError_t err, const char* what) {
  return fail(MOE_ERR_CUDA, "%s: %s", what, cudaGetErrorString(err));
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int num_sms_current() {
  static std::atomic<int> cached[64];  // zero-initialised (static storage)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

int32_t* status_word(void* ws) { return reinterpret_cast<int32_t*>(ws); }

// Per-chunk histograms of the plan: up to 256 chunks of E + 1 ints.
size_t plan_scratch_bytes(int32_t E) { return align256(size_t(256) * size_t(E + 1) * 4); }

int32_t* plan_scratch(void* ws) {
  return reinterpret_cast<int32_t*>(static_cast<uint8_t*>(ws) + kCtrlBytes);
}

// Intermediates of moe_ffn_fused inside the workspace.
struct FusedLayout {
  size_t xp, h, yk, w_sorted, inv, sync, total;
};

FusedLayout fused_layout(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  const int64_t R = M * topk;
  FusedLayout L;
  size_t off = kCtrlBytes + plan_scratch_bytes(E);
  L.xp = off;
  off += align256(size_t(R) * size_t(H) * 2);
  L.h = off;
  off += align256(size_t(R) * size_t(F) * 2);
  L.yk = off;  // fp32: the weighted rows are summed once more before the bf16 cast
  off += align256(size_t(R) * size_t(H) * 4);
  L.w_sorted = off;
  off += align256(size_t(R) * 4);
  L.inv = off;  // slot of every routed row (token-order dispatch)
  off += align256(size_t(R) * 4);
  L.sync = off;  // flags and counters of the single-kernel layer
  off += align256(moe::layer_sync_bytes(M, R, E));
  L.total = off;
  return L;
}

// moe_ffn_fused_fp8: the bf16 layout, then the quantised h and its row scales.
struct Fp8Layout {
  FusedLayout base;
  size_t hq, hs, total;
};

Fp8Layout fp8_layout(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  const int64_t R = M * topk;
  Fp8Layout L;
  L.base = fused_layout(M, H, F, E, topk);
  size_t off = L.base.total;
  L.hq = off;
  off += align256(size_t(R) * size_t(F));
  L.hs = off;
  off += align256(size_t(R) * 4);
  L.total = off;
  return L;
}

// moe_grouped_gemm_mx: the control block, then the A and B scale groups.
struct GemmMxLayout {
  size_t sfa, sfb, total;
};

GemmMxLayout gemm_mx_layout(int64_t R, int64_t N, int64_t K, int32_t E) {
  GemmMxLayout L;
  size_t off = kCtrlBytes;
  L.sfa = off;
  off += align256(moe::mx_sfa_bytes(R, E, K));
  L.sfb = off;
  off += align256(moe::mx_sfb_bytes(E, N, K));
  L.total = off;
  return L;
}

// moe_ffn_fused_mx: plan scratch, the dispatched rows, the E4M3 codes of h and
// their scale groups (written by GEMM1's epilogue), the weights' scale groups, the
// weighted rows (fp32), sorted gate weights and the token-order slots.
struct MxLayout {
  size_t xp, hq, sfa, sfb, yk, w_sorted, inv, total;
};

MxLayout mx_layout(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  const int64_t R = M * topk;
  MxLayout L;
  size_t off = kCtrlBytes + plan_scratch_bytes(E);
  L.xp = off;
  off += align256(size_t(R) * size_t(H) * 2);
  L.hq = off;
  off += align256(size_t(R) * size_t(F));
  L.sfa = off;
  off += align256(moe::mx_sfa_bytes(R, E, F));
  L.sfb = off;
  off += align256(moe::mx_sfb_bytes(E, H, F));
  L.yk = off;
  off += align256(size_t(R) * size_t(H) * 4);
  L.w_sorted = off;
  off += align256(size_t(R) * 4);
  L.inv = off;
  off += align256(size_t(R) * 4);
  L.total = off;
  return L;
}

moe_status check_ws(moe_op op, void* ws, size_t ws_bytes, int64_t M, int64_t H, int64_t F,
                    int32_t E, int32_t topk) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(MOE_ERR_MISALIGNED, "workspace must be 256-byte aligned");
  const size_t need = moe_workspace_size(op, M, H, F, E, topk);
  if (ws_bytes < need)
    return fail(MOE_ERR_WORKSPACE_TOO_SMALL, "workspace has %zu bytes, needs %zu", ws_bytes, need);
  return MOE_OK;
}

moe_status check_route(int64_t M, int32_t E, int32_t topk) {
  if (M < 0) return fail(MOE_ERR_INVALID_ARG, "M = %lld < 0", (long long)M);
  if (E < 1) return fail(MOE_ERR_INVALID_ARG, "E = %d < 1", E);
  if (E > MOE_MAX_EXPERTS)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d > %d", E, MOE_MAX_EXPERTS);
  if (topk < 1 || topk > E) return fail(MOE_ERR_INVALID_ARG, "topk = %d not in [1, E=%d]", topk, E);
  if (topk > 32) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "topk = %d > 32", topk);
  if (M > kMaxRows / topk) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "M*topk exceeds 2^31-1");
  return MOE_OK;
}

}  // namespace

namespace moe {
// Used by entry points defined in other files of the library.
moe_status record_error(moe_status st, const std::string& msg) {
  g_last_error = msg;
  return st;
}
void clear_last_error() { g_last_error.clear(); }
uint64_t wait_timeout_ns() { return g_timeout_ns; }

// The shape checks of the whole layer (moe_ffn_fused and its variants): the
// routing sizes, H and F positive multiples of 64, and every row count that the
// kernels hold in int32 within range.  Records the message; returns the status.
moe_status check_layer_shape(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  moe_status st = check_route(M, E, topk);
  if (st != MOE_OK) return st;
  if (H <= 0 || H % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H = %lld must be a positive multiple of 64", (long long)H);
  if (F <= 0 || F % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "F = %lld must be a positive multiple of 64", (long long)F);
  if (H > (int64_t(1) << 30) || F > (int64_t(1) << 29) || int64_t(E) * H > kMaxRows || int64_t(E) * F > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H or F too large");
  return MOE_OK;
}
}  // namespace moe

extern "C" {

int moe_abi_version(void) { return 1; }

const char* moe_last_error(void) { return g_last_error.c_str(); }

void moe_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns > 0 ? ns : 1; }

moe_status moe_set_stage_events(void* const* events) {
  g_last_error.clear();
  if (events == nullptr) {
    g_stage_events_on = false;
    return MOE_OK;
  }
  for (int i = 0; i < 6; ++i) g_stage_events[i] = static_cast<cudaEvent_t>(events[i]);
  g_stage_events_on = true;
  return MOE_OK;
}

moe_status moe_set_fault_injection(int32_t kind, int32_t index) {
  if (kind == 0) {
    g_withhold_mtile = -1;
    return MOE_OK;
  }
  if (kind == 1 && index >= 0) {
    g_withhold_mtile = index;
    return MOE_OK;
  }
  return fail(MOE_ERR_INVALID_ARG, "unknown fault injection kind %d", kind);
}

size_t moe_workspace_size(moe_op op, int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk) {
  if (M < 0 || H < 0 || F < 0 || topk < 0 || E < 1 || E > MOE_MAX_EXPERTS) return kCtrlBytes;
  // sizes whose byte counts could overflow are never valid: no workspace is enough
  if ((topk > 0 && M > kMaxRows / topk) || H > (int64_t(1) << 30) || F > (int64_t(1) << 30))
    return SIZE_MAX;
  if (op == MOE_OP_FFN_FUSED) return fused_layout(M, H, F, E, topk).total;
  if (op == MOE_OP_FFN_FP8) return fp8_layout(M, H, F, E, topk).total;
  if (op == MOE_OP_FFN_MX) return mx_layout(M, H, F, E, topk).total;
  if (op == MOE_OP_GEMM_MX) return gemm_mx_layout(M, H, F, E).total;
  if (op == MOE_OP_PLAN) return kCtrlBytes + plan_scratch_bytes(E);
  return kCtrlBytes;
}

moe_status moe_get_device_status(void* ws, void* stream) {
  if (ws == nullptr) return fail(MOE_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t v = 0;
  cudaError_t err = cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, s);
  // the whole control block: status word and the GEMM tile queue
  if (err == cudaSuccess) err = cudaMemsetAsync(ws, 0, kCtrlBytes, s);
  if (err == cudaSuccess) err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_get_device_status");
  return static_cast<moe_status>(v);
}

moe_status moe_plan(const int32_t* topk_ids, const float* topk_w, int64_t M, int32_t E,
                    int32_t topk, int32_t* counts, int32_t* offsets, int32_t* perm,
                    int32_t* inv_perm, float* w_sorted, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  moe_status st = check_route(M, E, topk);
  if (st != MOE_OK) return st;
  if (counts == nullptr || offsets == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (M > 0 && (topk_ids == nullptr || perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "topk_ids and perm must not be NULL");
  if (w_sorted != nullptr && topk_w == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "w_sorted requested without topk_w");
  st = check_ws(MOE_OP_PLAN, ws, ws_bytes, M, 0, 0, E, topk);
  if (st != MOE_OK) return st;
  cudaError_t err = moe::launch_plan(topk_ids, topk_w, static_cast<int32_t>(M * topk), E, counts,
                                     offsets, perm, inv_perm, w_sorted, status_word(ws),
                                     plan_scratch(ws), num_sms_current(),
                                     reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_plan launch");
  return MOE_OK;
}

moe_status moe_route(const float* logits, int64_t M, int32_t E, int32_t topk, int32_t* topk_ids,
                     float* topk_w, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  moe_status st = check_route(M, E, topk);
  if (st != MOE_OK) return st;
  st = check_ws(MOE_OP_ROUTE, ws, ws_bytes, M, 0, 0, E, topk);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (logits == nullptr || topk_ids == nullptr || topk_w == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "logits, topk_ids and topk_w must not be NULL");
  cudaError_t err = moe::launch_route(logits, M, E, topk, topk_ids, topk_w, num_sms_current(),
                                      reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_route launch");
  return MOE_OK;
}

moe_status moe_route_plan(const float* logits, int64_t M, int32_t E, int32_t topk,
                          int32_t* topk_ids, float* topk_w, int32_t* counts, int32_t* offsets,
                          int32_t* perm, int32_t* inv_perm, float* w_sorted, void* ws,
                          size_t ws_bytes, void* stream) {
  g_last_error.clear();
  moe_status st = check_route(M, E, topk);
  if (st != MOE_OK) return st;
  st = check_ws(MOE_OP_PLAN, ws, ws_bytes, M, 0, 0, E, topk);
  if (st != MOE_OK) return st;
  if (counts == nullptr || offsets == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (M > 0 && (logits == nullptr || topk_ids == nullptr || topk_w == nullptr || perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "logits, topk_ids, topk_w and perm must not be NULL");
  cudaError_t err = moe::launch_route_plan(logits, M, E, topk, topk_ids, topk_w, counts, offsets,
                                           perm, inv_perm, w_sorted, status_word(ws),
                                           plan_scratch(ws), num_sms_current(),
                                           reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_route_plan launch");
  return MOE_OK;
}

moe_status moe_dispatch(const void* x, const int32_t* perm, int64_t M, int64_t H, int32_t topk,
                        void* xp, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (M < 0 || topk < 1 || topk > 32 || M > kMaxRows / topk)
    return fail(MOE_ERR_INVALID_ARG, "bad M=%lld or topk=%d", (long long)M, topk);
  if (H <= 0 || H % 8 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H = %lld must be a positive multiple of 8", (long long)H);
  moe_status st = check_ws(MOE_OP_DISPATCH, ws, ws_bytes, M, H, 0, 1, topk);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (x == nullptr || perm == nullptr || xp == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "x, perm and xp must not be NULL");
  if (!aligned16(x) || !aligned16(xp)) return fail(MOE_ERR_MISALIGNED, "x and xp must be 16-byte aligned");
  cudaError_t err = moe::launch_dispatch(x, perm, M, H, topk, xp, status_word(ws), num_sms_current(),
                                         reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_dispatch launch");
  return MOE_OK;
}

moe_status moe_combine(const void* y, int32_t y_fp32, const int32_t* inv_perm,
                       const float* topk_w, int64_t M, int64_t H, int32_t topk, void* out,
                       void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (M < 0 || topk < 1 || topk > 32 || M > kMaxRows / topk)
    return fail(MOE_ERR_INVALID_ARG, "bad M=%lld or topk=%d", (long long)M, topk);
  if (H <= 0 || H % 8 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H = %lld must be a positive multiple of 8", (long long)H);
  moe_status st = check_ws(MOE_OP_COMBINE, ws, ws_bytes, M, H, 0, 1, topk);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (y == nullptr || out == nullptr) return fail(MOE_ERR_INVALID_ARG, "y and out must not be NULL");
  if (!aligned16(y) || !aligned16(out)) return fail(MOE_ERR_MISALIGNED, "y and out must be 16-byte aligned");
  if (y_fp32 != 0 && y_fp32 != 1) return fail(MOE_ERR_INVALID_ARG, "y_fp32 must be 0 or 1");
  cudaError_t err = moe::launch_combine(y, y_fp32 != 0, inv_perm, topk_w, M, H, topk, out,
                                        status_word(ws), num_sms_current(),
                                        reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_combine launch");
  return MOE_OK;
}

moe_status moe_combine_add(const void* y, int32_t y_fp32, const int32_t* inv_perm,
                           const float* topk_w, const void* add, float alpha, float beta,
                           int64_t M, int64_t H, int32_t topk, void* out, void* ws,
                           size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (M < 0 || topk < 1 || topk > 32 || M > kMaxRows / topk)
    return fail(MOE_ERR_INVALID_ARG, "bad M=%lld or topk=%d", (long long)M, topk);
  if (H <= 0 || H % 8 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "H = %lld must be a positive multiple of 8", (long long)H);
  moe_status st = check_ws(MOE_OP_COMBINE, ws, ws_bytes, M, H, 0, 1, topk);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (y == nullptr || out == nullptr) return fail(MOE_ERR_INVALID_ARG, "y and out must not be NULL");
  if (add == nullptr && beta != 0.0f) return fail(MOE_ERR_INVALID_ARG, "add is NULL but beta != 0");
  if (!aligned16(y) || !aligned16(out) || !aligned16(add))
    return fail(MOE_ERR_MISALIGNED, "y, out and add must be 16-byte aligned");
  if (y_fp32 != 0 && y_fp32 != 1) return fail(MOE_ERR_INVALID_ARG, "y_fp32 must be 0 or 1");
  cudaError_t err = moe::launch_combine_add(y, y_fp32 != 0, inv_perm, topk_w, add, alpha, beta,
                                            M, H, topk, out, status_word(ws), num_sms_current(),
                                            reinterpret_cast<cudaStream_t>(stream));
  if (err != cudaSuccess) return cuda_fail(err, "moe_combine_add launch");
  return MOE_OK;
}

moe_status moe_grouped_gemm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                            int64_t R, int64_t K, int64_t N, moe_epilogue epi,
                            const float* w_sorted, const int32_t* perm, void* C, void* ws,
                            size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64", (long long)K);
  if (N <= 0 || N % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "N = %lld must be a positive multiple of 64", (long long)N);
  if (epi != MOE_EPI_STORE && epi != MOE_EPI_SWIGLU && epi != MOE_EPI_WEIGHT_SCATTER)
    return fail(MOE_ERR_INVALID_ARG, "unknown epilogue %d", (int)epi);
  if (epi == MOE_EPI_SWIGLU && (N / 2) % 64 != 0)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "SWIGLU needs N/2 = %lld a multiple of 64", (long long)(N / 2));
  if (K > (int64_t(1) << 30) || N > (int64_t(1) << 30) || E * K > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N too large");
  moe_status st = check_ws(MOE_OP_GROUPED_GEMM, ws, ws_bytes, R, N, K, E, 1);
  if (st != MOE_OK) return st;
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets must not be NULL");
  if (R == 0) return MOE_OK;
  if (A == nullptr || B == nullptr || C == nullptr) return fail(MOE_ERR_INVALID_ARG, "A, B and C must not be NULL");
  if (!aligned16(A) || !aligned16(B) || !aligned16(C)) return fail(MOE_ERR_MISALIGNED, "A, B and C must be 16-byte aligned");
  if (epi == MOE_EPI_WEIGHT_SCATTER && (w_sorted == nullptr || perm == nullptr))
    return fail(MOE_ERR_INVALID_ARG, "WEIGHT_SCATTER needs w_sorted and perm");
  const int rc = moe::launch_grouped_gemm(A, B, offsets, E, R, K, N, static_cast<int>(epi), w_sorted,
                                          perm, C, status_word(ws), g_timeout_ns, num_sms_current(),
                                          reinterpret_cast<cudaStream_t>(stream));
  if (rc == 1) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  if (rc != 0) return cuda_fail(cudaGetLastError(), "moe_grouped_gemm launch");
  return MOE_OK;
}

}  // extern "C"

namespace {

// The layer (moe_ffn_fused and moe_ffn_fused_add).  n_c as moe_ffn_fused; the
// combine applies out = bf16(alpha * sum + beta * add) (alpha = 1, beta = 0: the
// plain layer, add unused).
moe_status ffn_fused_impl(const void* x, const void* W1, const void* W2, const int32_t* topk_ids,
                          const float* topk_w, const void* add, float alpha, float beta,
                          int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk, int32_t n_c,
                          void* out, int32_t* counts, int32_t* offsets, int32_t* perm, void* ws,
                          size_t ws_bytes, void* stream) {
  g_last_error.clear();
  moe_status st = moe::check_layer_shape(M, H, F, E, topk);
  if (st != MOE_OK) return st;
  if (n_c < -1) return fail(MOE_ERR_INVALID_ARG, "n_c = %d < -1", n_c);
  st = check_ws(MOE_OP_FFN_FUSED, ws, ws_bytes, M, H, F, E, topk);
  if (st != MOE_OK) return st;
  if (counts == nullptr || offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (M == 0) {
    // Still a defined plan: zero counts and offsets.
    cudaStream_t s0 = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t err = moe::launch_plan(topk_ids, topk_w, 0, E, counts, offsets, perm, nullptr,
                                       nullptr, status_word(ws), plan_scratch(ws),
                                       num_sms_current(), s0);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_ffn_fused plan");
  }
  if (x == nullptr || W1 == nullptr || W2 == nullptr || topk_ids == nullptr || topk_w == nullptr ||
      out == nullptr || perm == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "x, W1, W2, topk_ids, topk_w, out and perm must not be NULL");
  if (!aligned16(x) || !aligned16(W1) || !aligned16(W2) || !aligned16(out))
    return fail(MOE_ERR_MISALIGNED, "x, W1, W2 and out must be 16-byte aligned");
  const bool gemm_add = alpha != 1.0f || beta != 0.0f;
  if (gemm_add && beta != 0.0f && add == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "add is NULL but beta != 0");
  if (gemm_add && !aligned16(add)) return fail(MOE_ERR_MISALIGNED, "add must be 16-byte aligned");

  const int64_t R = M * topk;
  // Overlapping kernel boundaries pays off on small layers only (measured).
  moe::PdlScope pdl(static_cast<double>(R) * static_cast<double>(H) * static_cast<double>(F) <
                    4294967296.0);
  const FusedLayout L = fused_layout(M, H, F, E, topk);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* xp = base + L.xp;
  void* h = base + L.h;
  void* yk = base + L.yk;
  float* w_sorted = reinterpret_cast<float*>(base + L.w_sorted);
  int32_t* status = status_word(ws);
  const int sms = num_sms_current();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  stage_mark(0, s);
  int32_t* inv = reinterpret_cast<int32_t*>(base + L.inv);
  cudaError_t err = moe::launch_plan(topk_ids, topk_w, static_cast<int32_t>(R), E, counts, offsets,
                                     perm, inv, w_sorted, status, plan_scratch(ws), sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused plan");
  stage_mark(1, s);
  const int32_t nc = gemm_add ? 0 : (n_c < 0 ? moe::profiled_n_c(M, H, F, E, topk) : n_c);
  if (nc > 0) {
    // One persistent kernel: nc memory CTAs (dispatch, combine) beside the GEMM CTAs.
    if (nc > 64 || nc >= sms) return fail(MOE_ERR_INVALID_ARG, "n_c = %d must be < min(65, #SMs = %d)", nc, sms);
    const int rc = moe::launch_moe_layer(x, W1, W2, perm, w_sorted, offsets, xp, h, yk, out, M, H, F,
                                         E, topk, nc, status, base + L.sync, g_timeout_ns,
                                         g_withhold_mtile, sms, s);
    if (rc == 1) return fail(MOE_ERR_CUDA, "tensor map encode failed (layer kernel)");
    if (rc == 3) return fail(MOE_ERR_CUDA, "cooperative launch refused: the layer kernel needs one co-resident CTA per SM");
    if (rc != 0) return cuda_fail(cudaGetLastError(), "moe_ffn_fused layer kernel");
    for (int i = 2; i <= 5; ++i) stage_mark(i, s);
    return MOE_OK;
  }
  err = moe::launch_dispatch_tokens(x, inv, M, H, topk, xp, status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused dispatch");
  stage_mark(2, s);
  int rc = moe::launch_grouped_gemm(xp, W1, offsets, E, R, H, 2 * F, MOE_EPI_SWIGLU, nullptr,
                                    nullptr, h, status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (GEMM1)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused GEMM1");
  stage_mark(3, s);
  rc = moe::launch_grouped_gemm(h, W2, offsets, E, R, F, H, MOE_EPI_WEIGHT_SCATTER, w_sorted, perm,
                                yk, status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (GEMM2)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused GEMM2");
  stage_mark(4, s);
  err = moe::launch_combine_add(yk, true, nullptr, nullptr, add, alpha, beta, M, H, topk, out,
                                status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused combine");
  stage_mark(5, s);
  return MOE_OK;
}

}  // namespace

extern "C" {

moe_status moe_ffn_fused(const void* x, const void* W1, const void* W2, const int32_t* topk_ids,
                         const float* topk_w, int64_t M, int64_t H, int64_t F, int32_t E,
                         int32_t topk, int32_t n_c, void* out, int32_t* counts,
                         int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes,
                         void* stream) {
  return ffn_fused_impl(x, W1, W2, topk_ids, topk_w, nullptr, 1.0f, 0.0f, M, H, F, E, topk, n_c,
                        out, counts, offsets, perm, ws, ws_bytes, stream);
}

moe_status moe_ffn_fused_add(const void* x, const void* W1, const void* W2,
                             const int32_t* topk_ids, const float* topk_w, const void* add,
                             float alpha, float beta, int64_t M, int64_t H, int64_t F, int32_t E,
                             int32_t topk, void* out, int32_t* counts, int32_t* offsets,
                             int32_t* perm, void* ws, size_t ws_bytes, void* stream) {
  return ffn_fused_impl(x, W1, W2, topk_ids, topk_w, add, alpha, beta, M, H, F, E, topk, 0, out,
                        counts, offsets, perm, ws, ws_bytes, stream);
}

moe_status moe_quantize_weights_e4m3(const void* W, int32_t E, int64_t K, int64_t N, void* Wq,
                                     float* scale, void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (K <= 0 || K % 16 != 0 || N <= 0 || N % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld and N = %lld must be positive multiples of 16", (long long)K, (long long)N);
  if (K > kMaxRows || N > kMaxRows || int64_t(E) * N > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N too large");
  if (W == nullptr || Wq == nullptr || scale == nullptr) return fail(MOE_ERR_INVALID_ARG, "W, Wq and scale must not be NULL");
  if (!aligned16(W) || !aligned16(Wq)) return fail(MOE_ERR_MISALIGNED, "W and Wq must be 16-byte aligned");
  const cudaError_t err = moe::launch_quantize_cols(W, E, K, N, Wq, scale, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_weights_e4m3");
}

moe_status moe_quantize_rows_e4m3(const void* A, int64_t R, int64_t K, void* Aq, float* scale,
                                  void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 64 != 0 || K > 32768)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64, at most 32768", (long long)K);
  moe_status st = check_ws(MOE_OP_GROUPED_GEMM, ws, ws_bytes, R, K, K, 1, 1);
  if (st != MOE_OK) return st;
  if (R == 0) return MOE_OK;
  if (A == nullptr || Aq == nullptr || scale == nullptr) return fail(MOE_ERR_INVALID_ARG, "A, Aq and scale must not be NULL");
  if (!aligned16(A) || !aligned16(Aq)) return fail(MOE_ERR_MISALIGNED, "A and Aq must be 16-byte aligned");
  const cudaError_t err = moe::launch_quantize_rows(A, R, K, Aq, scale, num_sms_current(),
                                                    reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_rows_e4m3");
}

moe_status moe_grouped_gemm_e4m3(const void* Aq, const float* a_scale, const void* BqT,
                                 const float* b_scale, const int32_t* offsets, int32_t E,
                                 int64_t R, int64_t K, int64_t N, const float* w_sorted,
                                 const int32_t* perm, float* C, void* ws, size_t ws_bytes,
                                 void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64", (long long)K);
  if (N <= 0 || N % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "N = %lld must be a positive multiple of 64", (long long)N);
  if (K > (int64_t(1) << 30) || N > (int64_t(1) << 30) || int64_t(E) * N > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N too large");
  moe_status st = check_ws(MOE_OP_GROUPED_GEMM, ws, ws_bytes, R, N, K, E, 1);
  if (st != MOE_OK) return st;
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets must not be NULL");
  if (R == 0) return MOE_OK;
  if (Aq == nullptr || BqT == nullptr || C == nullptr || a_scale == nullptr || b_scale == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "Aq, a_scale, BqT, b_scale and C must not be NULL");
  if (!aligned16(Aq) || !aligned16(BqT) || !aligned16(C))
    return fail(MOE_ERR_MISALIGNED, "Aq, BqT and C must be 16-byte aligned");
  const int rc = moe::launch_grouped_gemm_e4m3(Aq, a_scale, BqT, b_scale, offsets, E, R, K, N,
                                               w_sorted, perm, C, status_word(ws), g_timeout_ns,
                                               num_sms_current(),
                                               reinterpret_cast<cudaStream_t>(stream));
  if (rc == 1) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  if (rc != 0) return cuda_fail(cudaGetLastError(), "moe_grouped_gemm_e4m3 launch");
  return MOE_OK;
}

moe_status moe_ffn_fused_fp8(const void* x, const void* W1, const void* W2q,
                             const float* w2_scale, const int32_t* topk_ids, const float* topk_w,
                             int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk, void* out,
                             int32_t* counts, int32_t* offsets, int32_t* perm, void* ws,
                             size_t ws_bytes, void* stream) {
  g_last_error.clear();
  moe_status st = moe::check_layer_shape(M, H, F, E, topk);
  if (st != MOE_OK) return st;
  if (F > 32768) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "F = %lld must be at most 32768", (long long)F);
  st = check_ws(MOE_OP_FFN_FP8, ws, ws_bytes, M, H, F, E, topk);
  if (st != MOE_OK) return st;
  if (counts == nullptr || offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms_current();
  if (M == 0) {
    cudaError_t err = moe::launch_plan(topk_ids, topk_w, 0, E, counts, offsets, perm, nullptr,
                                       nullptr, status_word(ws), plan_scratch(ws), sms, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_ffn_fused_fp8 plan");
  }
  if (x == nullptr || W1 == nullptr || W2q == nullptr || w2_scale == nullptr || topk_ids == nullptr ||
      topk_w == nullptr || out == nullptr || perm == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "x, W1, W2q, w2_scale, topk_ids, topk_w, out and perm must not be NULL");
  if (!aligned16(x) || !aligned16(W1) || !aligned16(W2q) || !aligned16(out))
    return fail(MOE_ERR_MISALIGNED, "x, W1, W2q and out must be 16-byte aligned");
  const int64_t R = M * topk;
  moe::PdlScope pdl(static_cast<double>(R) * static_cast<double>(H) * static_cast<double>(F) <
                    4294967296.0);
  const Fp8Layout L = fp8_layout(M, H, F, E, topk);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* xp = base + L.base.xp;
  void* h = base + L.base.h;
  float* yk = reinterpret_cast<float*>(base + L.base.yk);
  float* w_sorted = reinterpret_cast<float*>(base + L.base.w_sorted);
  void* hq = base + L.hq;
  float* hs = reinterpret_cast<float*>(base + L.hs);
  int32_t* status = status_word(ws);

  int32_t* inv = reinterpret_cast<int32_t*>(base + L.base.inv);
  cudaError_t err = moe::launch_plan(topk_ids, topk_w, static_cast<int32_t>(R), E, counts, offsets,
                                     perm, inv, w_sorted, status, plan_scratch(ws), sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_fp8 plan");
  err = moe::launch_dispatch_tokens(x, inv, M, H, topk, xp, status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_fp8 dispatch");
  int rc = moe::launch_grouped_gemm(xp, W1, offsets, E, R, H, 2 * F, MOE_EPI_SWIGLU, nullptr,
                                    nullptr, h, status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (GEMM1)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused_fp8 GEMM1");
  err = moe::launch_quantize_rows(h, R, F, hq, hs, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_fp8 quantise");
  rc = moe::launch_grouped_gemm_e4m3(hq, hs, W2q, w2_scale, offsets, E, R, F, H, w_sorted, perm,
                                     yk, status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (FP8 GEMM2)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused_fp8 GEMM2");
  err = moe::launch_combine(yk, true, nullptr, nullptr, M, H, topk, out, status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_fp8 combine");
  return MOE_OK;
}

moe_status moe_quantize_weights_mx(const void* W, int32_t E, int64_t K, int64_t N, void* BqT,
                                   uint8_t* sf, void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (K <= 0 || K % 32 != 0 || N <= 0 || N % 16 != 0)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 32 and N = %lld of 16", (long long)K, (long long)N);
  if (K > kMaxRows || N > kMaxRows || int64_t(E) * N > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N too large");
  if (W == nullptr || BqT == nullptr || sf == nullptr) return fail(MOE_ERR_INVALID_ARG, "W, BqT and sf must not be NULL");
  if (!aligned16(W) || !aligned16(BqT)) return fail(MOE_ERR_MISALIGNED, "W and BqT must be 16-byte aligned");
  const cudaError_t err = moe::launch_quantize_weights_mx(W, E, K, N, BqT, sf, num_sms_current(),
                                                          reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_weights_mx");
}

moe_status moe_quantize_rows_mx(const void* A, int64_t R, int64_t K, void* Aq, uint8_t* sf,
                                void* stream) {
  g_last_error.clear();
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 32 != 0 || K > (int64_t(1) << 30))
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 32", (long long)K);
  if (R == 0) return MOE_OK;
  if (A == nullptr || Aq == nullptr || sf == nullptr) return fail(MOE_ERR_INVALID_ARG, "A, Aq and sf must not be NULL");
  if (!aligned16(A) || !aligned16(Aq)) return fail(MOE_ERR_MISALIGNED, "A and Aq must be 16-byte aligned");
  const cudaError_t err = moe::launch_quantize_rows_mx(A, R, K, Aq, sf, num_sms_current(),
                                                       reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_quantize_rows_mx");
}

moe_status moe_grouped_gemm_swiglu_mx(const void* A, const void* B, const int32_t* offsets,
                                      int32_t E, int64_t R, int64_t K, int64_t N2, void* hq,
                                      uint8_t* h_sf, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 64", (long long)K);
  if (N2 <= 0 || N2 % 128 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "N2 = %lld must be a positive multiple of 128", (long long)N2);
  if (K > (int64_t(1) << 30) || N2 > (int64_t(1) << 30) || E * K > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N2 too large");
  moe_status st = check_ws(MOE_OP_GROUPED_GEMM, ws, ws_bytes, R, N2, K, E, 1);
  if (st != MOE_OK) return st;
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets must not be NULL");
  if (R == 0) return MOE_OK;
  if (A == nullptr || B == nullptr || hq == nullptr || h_sf == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "A, B, hq and h_sf must not be NULL");
  if (!aligned16(A) || !aligned16(B) || !aligned16(hq)) return fail(MOE_ERR_MISALIGNED, "A, B and hq must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(h_sf) & 1u) != 0) return fail(MOE_ERR_MISALIGNED, "h_sf must be 2-byte aligned");
  const int rc = moe::launch_grouped_gemm_swiglu_mx(A, B, offsets, E, R, K, N2, static_cast<uint8_t*>(hq),
                                                    h_sf, true, 0, status_word(ws), g_timeout_ns,
                                                    num_sms_current(), reinterpret_cast<cudaStream_t>(stream));
  if (rc == 1) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  if (rc != 0) return cuda_fail(cudaGetLastError(), "moe_grouped_gemm_swiglu_mx launch");
  return MOE_OK;
}

moe_status moe_grouped_gemm_mx(const void* Aq, const uint8_t* a_sf, const void* BqT,
                               const uint8_t* b_sf, const int32_t* offsets, int32_t E, int64_t R,
                               int64_t K, int64_t N, const float* w_sorted, const int32_t* perm,
                               float* C, void* ws, size_t ws_bytes, void* stream) {
  g_last_error.clear();
  if (E < 1 || E > MOE_MAX_EXPERTS) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "E = %d not in [1, %d]", E, MOE_MAX_EXPERTS);
  if (R < 0 || R > kMaxRows) return fail(MOE_ERR_INVALID_ARG, "R = %lld out of range", (long long)R);
  if (K <= 0 || K % 32 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K = %lld must be a positive multiple of 32", (long long)K);
  if (N <= 0 || N % 64 != 0) return fail(MOE_ERR_UNSUPPORTED_SHAPE, "N = %lld must be a positive multiple of 64", (long long)N);
  if (K > (int64_t(1) << 30) || N > (int64_t(1) << 30) || int64_t(E) * N > kMaxRows)
    return fail(MOE_ERR_UNSUPPORTED_SHAPE, "K or N too large");
  moe_status st = check_ws(MOE_OP_GEMM_MX, ws, ws_bytes, R, N, K, E, 1);
  if (st != MOE_OK) return st;
  if (offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "offsets must not be NULL");
  if (R == 0) return MOE_OK;
  if (Aq == nullptr || BqT == nullptr || C == nullptr || a_sf == nullptr || b_sf == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "Aq, a_sf, BqT, b_sf and C must not be NULL");
  if (!aligned16(Aq) || !aligned16(BqT) || !aligned16(C))
    return fail(MOE_ERR_MISALIGNED, "Aq, BqT and C must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const GemmMxLayout L = gemm_mx_layout(R, N, K, E);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int sms = num_sms_current();
  cudaError_t err = moe::launch_pack_sfa(a_sf, offsets, E, R, K, base + L.sfa, status_word(ws), sms, s);
  if (err == cudaSuccess) err = moe::launch_pack_sfb(b_sf, E, N, K, base + L.sfb, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_grouped_gemm_mx scale packing");
  const int rc = moe::launch_grouped_gemm_mx(Aq, base + L.sfa, BqT, base + L.sfb, offsets, E, R, K, N,
                                             w_sorted, perm, C, status_word(ws), g_timeout_ns, sms, s);
  if (rc == 1) return fail(MOE_ERR_CUDA, "cuTensorMapEncodeTiled failed (driver entry point or arguments)");
  if (rc != 0) return cuda_fail(cudaGetLastError(), "moe_grouped_gemm_mx launch");
  return MOE_OK;
}

moe_status moe_ffn_fused_mx(const void* x, const void* W1, const void* W2q, const uint8_t* w2_sf,
                            const int32_t* topk_ids, const float* topk_w, int64_t M, int64_t H,
                            int64_t F, int32_t E, int32_t topk, void* out, int32_t* counts,
                            int32_t* offsets, int32_t* perm, void* ws, size_t ws_bytes,
                            void* stream) {
  g_last_error.clear();
  moe_status st = moe::check_layer_shape(M, H, F, E, topk);
  if (st != MOE_OK) return st;
  st = check_ws(MOE_OP_FFN_MX, ws, ws_bytes, M, H, F, E, topk);
  if (st != MOE_OK) return st;
  if (counts == nullptr || offsets == nullptr) return fail(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = num_sms_current();
  if (M == 0) {
    cudaError_t err = moe::launch_plan(topk_ids, topk_w, 0, E, counts, offsets, perm, nullptr,
                                       nullptr, status_word(ws), plan_scratch(ws), sms, s);
    return err == cudaSuccess ? MOE_OK : cuda_fail(err, "moe_ffn_fused_mx plan");
  }
  if (x == nullptr || W1 == nullptr || W2q == nullptr || w2_sf == nullptr || topk_ids == nullptr ||
      topk_w == nullptr || out == nullptr || perm == nullptr)
    return fail(MOE_ERR_INVALID_ARG, "x, W1, W2q, w2_sf, topk_ids, topk_w, out and perm must not be NULL");
  if (!aligned16(x) || !aligned16(W1) || !aligned16(W2q) || !aligned16(out))
    return fail(MOE_ERR_MISALIGNED, "x, W1, W2q and out must be 16-byte aligned");
  const int64_t R = M * topk;
  moe::PdlScope pdl(static_cast<double>(R) * static_cast<double>(H) * static_cast<double>(F) <
                    4294967296.0);
  const MxLayout L = mx_layout(M, H, F, E, topk);
  uint8_t* base = static_cast<uint8_t*>(ws);
  void* xp = base + L.xp;
  uint8_t* hq = base + L.hq;
  uint8_t* sfa = base + L.sfa;
  uint8_t* sfb = base + L.sfb;
  float* yk = reinterpret_cast<float*>(base + L.yk);
  float* w_sorted = reinterpret_cast<float*>(base + L.w_sorted);
  int32_t* inv = reinterpret_cast<int32_t*>(base + L.inv);
  int32_t* status = status_word(ws);

  // stage events (moe_set_stage_events): the first stage holds the weight-scale
  // rearrangement and the plan
  stage_mark(0, s);
  cudaError_t err = moe::launch_pack_sfb(w2_sf, E, H, F, sfb, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_mx weight scales");
  err = moe::launch_plan(topk_ids, topk_w, static_cast<int32_t>(R), E, counts, offsets, perm, inv,
                         w_sorted, status, plan_scratch(ws), sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_mx plan");
  stage_mark(1, s);
  err = moe::launch_dispatch_tokens(x, inv, M, H, topk, xp, status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_mx dispatch");
  stage_mark(2, s);
  int rc = moe::launch_grouped_gemm_swiglu_mx(xp, W1, offsets, E, R, H, 2 * F, hq, sfa, false,
                                              moe::mx_kg_pad(F), status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (GEMM1)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused_mx GEMM1");
  stage_mark(3, s);
  rc = moe::launch_grouped_gemm_mx(hq, sfa, W2q, sfb, offsets, E, R, F, H, w_sorted, perm, yk,
                                   status, g_timeout_ns, sms, s);
  if (rc != 0) return rc == 1 ? fail(MOE_ERR_CUDA, "tensor map encode failed (MX GEMM2)")
                              : cuda_fail(cudaGetLastError(), "moe_ffn_fused_mx GEMM2");
  stage_mark(4, s);
  err = moe::launch_combine(yk, true, nullptr, nullptr, M, H, topk, out, status, sms, s);
  if (err != cudaSuccess) return cuda_fail(err, "moe_ffn_fused_mx combine");
  stage_mark(5, s);
  return MOE_OK;
}

}  // extern "C"
