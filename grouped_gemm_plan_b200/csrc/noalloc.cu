// noalloc.cu -- moe_ffn_fused_noalloc: the whole layer without any device
// allocation, its intermediates held in one fixed-size array of this library.
//
// Why it exists: some callers of this library cannot allocate device memory.
// A host program handed only input and output buffers (a C or plugin caller with
// no allocator of its own), or a process whose device memory was reserved up
// front by another allocator, cannot call cudaMalloc for the workspace that
// moe_ffn_fused needs -- the call would fail, or would stall the device at a bad
// time.  This entry point needs no workspace from the caller: the expert-ordered
// activations, the SwiGLU activations, the gate-weighted expert rows and the
// status word live in g_noalloc_scratch below, a file-scope device array that
// every GPU which loads this library holds until the process exits.
//
// It runs the same kernels as moe_ffn_fused (plan, dispatch, GEMM1+SwiGLU,
// GEMM2+scatter, combine) through the same launchers; only where the
// intermediates live differs.
#include <mutex>
#include <string>

#include "common.cuh"

namespace moe {
cudaError_t launch_plan(const int32_t* ids, const float* w, int32_t R, int32_t E, int32_t* counts,
                        int32_t* offsets, int32_t* perm, int32_t* inv, float* w_sorted,
                        int32_t* status, int32_t* scratch, int num_sms, cudaStream_t stream);
cudaError_t launch_dispatch(const void* x, const int32_t* perm, int64_t M, int64_t H, int32_t topk,
                            void* xp, int32_t* status, int num_sms, cudaStream_t stream);
cudaError_t launch_combine(const void* y, bool y_f32, const int32_t* inv, const float* w,
                           int64_t M, int64_t H, int32_t topk, void* out, int32_t* status,
                           int num_sms, cudaStream_t stream);
int launch_grouped_gemm(const void* A, const void* B, const int32_t* offsets, int32_t E,
                        int64_t R, int64_t K, int64_t N, int epi, const float* w_sorted,
                        const int32_t* perm, void* C, int32_t* status, uint64_t timeout_ns,
                        int num_sms, cudaStream_t stream);
moe_status record_error(moe_status st, const std::string& msg);
void clear_last_error();
moe_status check_layer_shape(int64_t M, int64_t H, int64_t F, int32_t E, int32_t topk);
uint64_t wait_timeout_ns();
}  // namespace moe

// The scratch.  Host code must never pass &g_noalloc_scratch to a kernel: on the
// host that name is a stand-in, not a device address.  The device address comes
// from cudaGetSymbolAddress, once per device (scratch_address below).
static __device__ __align__(256) uint8_t g_noalloc_scratch[MOE_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};
int g_num_sms[kMaxDevices] = {0};

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
  size_t hist, xp, h, yk, w_sorted, total;
};

// status word [0, 256), the plan's per-chunk histograms (256 x (E + 1) int32),
// then xp bf16 [R, H], h bf16 [R, F], yk fp32 [R, H], w_sorted fp32 [R]
Layout layout(int64_t R, int64_t H, int64_t F, int32_t E) {
  Layout L;
  size_t off = 256;
  L.hist = off;
  off += al256(size_t(256) * size_t(E + 1) * 4);
  L.xp = off;
  off += al256(size_t(R) * size_t(H) * 2);
  L.h = off;
  off += al256(size_t(R) * size_t(F) * 2);
  L.yk = off;
  off += al256(size_t(R) * size_t(H) * 4);
  L.w_sorted = off;
  off += al256(size_t(R) * 4);
  L.total = off;
  return L;
}

// Device address of the scratch on the current device, looked up on the first
// call for that device (with that device current) and remembered.
cudaError_t scratch_address(void** addr, int* sms) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (err != cudaSuccess) return err;
    int n = 0;
    err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (err != cudaSuccess) return err;
    g_scratch_addr[dev] = p;
    g_num_sms[dev] = n;
  }
  *addr = g_scratch_addr[dev];
  *sms = g_num_sms[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" moe_status moe_ffn_fused_noalloc(const void* x, const void* W1, const void* W2,
                                            const int32_t* topk_ids, const float* topk_w,
                                            int64_t M, int64_t H, int64_t F, int32_t E,
                                            int32_t topk, void* out, int32_t* counts,
                                            int32_t* offsets, int32_t* perm, int32_t* status,
                                            void* stream) {
  using moe::record_error;
  moe::clear_last_error();
  // The same shape checks, with the same status codes, as moe_ffn_fused; they also
  // bound R = M * topk and every size below, so the layout arithmetic cannot wrap.
  const moe_status shape = moe::check_layer_shape(M, H, F, E, topk);
  if (shape != MOE_OK) return shape;
  const int64_t R = M * topk;
  const Layout L = layout(R, H, F, E);
  if (L.total > size_t(MOE_NOALLOC_SCRATCH_BYTES))
    return record_error(MOE_ERR_WORKSPACE_TOO_SMALL,
                        "this shape needs " + std::to_string(L.total) +
                            " bytes of scratch; the library's static scratch holds " +
                            std::to_string(size_t(MOE_NOALLOC_SCRATCH_BYTES)) +
                            " (use moe_ffn_fused with a caller workspace)");
  if (counts == nullptr || offsets == nullptr)
    return record_error(MOE_ERR_INVALID_ARG, "counts and offsets must not be NULL");
  if (M > 0 && (x == nullptr || W1 == nullptr || W2 == nullptr || topk_ids == nullptr ||
                topk_w == nullptr || out == nullptr || perm == nullptr))
    return record_error(MOE_ERR_INVALID_ARG, "x, W1, W2, topk_ids, topk_w, out and perm must not be NULL");
  const auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (M > 0 && (!a16(x) || !a16(W1) || !a16(W2) || !a16(out)))
    return record_error(MOE_ERR_MISALIGNED, "x, W1, W2 and out must be 16-byte aligned");

  void* base = nullptr;
  int sms = 0;
  cudaError_t err = scratch_address(&base, &sms);
  if (err != cudaSuccess)
    return record_error(MOE_ERR_CUDA, std::string("scratch set-up: ") + cudaGetErrorString(err));
  uint8_t* b = static_cast<uint8_t*>(base);
  int32_t* st = reinterpret_cast<int32_t*>(b);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  // The array keeps the previous call's contents; only the status word must
  // start at zero.  On success every intermediate row is written before it is
  // read.  When the call ends with a device error (an expert id out of range:
  // the plan then leaves every expert empty), the GEMMs write no rows and the
  // combine reads rows left by an earlier call, so `out` is undefined whenever
  // the status is not MOE_OK.
  err = cudaMemsetAsync(st, 0, sizeof(int32_t), s);
  if (err == cudaSuccess)
    err = moe::launch_plan(topk_ids, topk_w, static_cast<int32_t>(R), E, counts, offsets, perm,
                           nullptr, reinterpret_cast<float*>(b + L.w_sorted), st,
                           reinterpret_cast<int32_t*>(b + L.hist), sms, s);
  if (err == cudaSuccess && R > 0)
    err = moe::launch_dispatch(x, perm, M, H, topk, b + L.xp, st, sms, s);
  if (err != cudaSuccess)
    return record_error(MOE_ERR_CUDA, std::string("plan/dispatch: ") + cudaGetErrorString(err));
  if (R > 0) {
    int rc = moe::launch_grouped_gemm(b + L.xp, W1, offsets, E, R, H, 2 * F, MOE_EPI_SWIGLU,
                                      nullptr, nullptr, b + L.h, st, moe::wait_timeout_ns(), sms,
                                      s);
    if (rc == 0)
      rc = moe::launch_grouped_gemm(b + L.h, W2, offsets, E, R, F, H, MOE_EPI_WEIGHT_SCATTER,
                                    reinterpret_cast<const float*>(b + L.w_sorted), perm, b + L.yk,
                                    st, moe::wait_timeout_ns(), sms, s);
    if (rc != 0)
      return record_error(MOE_ERR_CUDA, rc == 1 ? "tensor map encode failed"
                                                : cudaGetErrorString(cudaGetLastError()));
    err = moe::launch_combine(b + L.yk, true, nullptr, nullptr, M, H, topk, out, st, sms, s);
  }
  if (err == cudaSuccess && status != nullptr)
    err = cudaMemcpyAsync(status, st, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
  if (err != cudaSuccess)
    return record_error(MOE_ERR_CUDA, std::string("combine/status: ") + cudaGetErrorString(err));
  return MOE_OK;
}
