// Library-wide entry points (errors, device checks, status word) and host helpers.
#include <atomic>
#include <cstring>
#include <mutex>

#include "tg_host.h"

namespace tg {

static thread_local int g_last_cuda_error = 0;

void set_cuda_error(cudaError_t e) { g_last_cuda_error = static_cast<int>(e); }

int check_device() {
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  return tg_device_supported(dev) ? TG_OK : TG_ERR_UNSUPPORTED_DEVICE;
}

int check_launch() {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return TG_ERR_CUDA;
  }
  return TG_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

int make_tmap_bf16_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t ld, uint32_t box_cols, uint32_t box_rows) {
  return make_tmap_bf16_2d_swz(out, base, rows, cols, ld, box_cols, box_rows, true);
}

int make_tmap_bf16_2d_swz(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                          uint64_t ld, uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
  auto fn = encode_fn();
  if (!fn) {
    set_cuda_error(cudaErrorNotSupported);
    return TG_ERR_CUDA;
  }
  if (!aligned16(base) || (ld * 2) % 16 != 0) return TG_ERR_MISALIGNED;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                  strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_cuda_error(cudaErrorInvalidValue);
    return TG_ERR_INVALID_ARGUMENT;
  }
  return TG_OK;
}

namespace {
std::atomic<int> g_launch_overlap{1};
std::atomic<int> g_gather_tma{0};
std::atomic<int> g_scorer_pair{1};
}

bool gather_use_tma() { return g_gather_tma.load(std::memory_order_relaxed) != 0; }
bool scorer_use_pair() { return g_scorer_pair.load(std::memory_order_relaxed) != 0; }

bool launch_overlap() { return g_launch_overlap.load(std::memory_order_relaxed) != 0; }
void set_launch_overlap(bool on) { g_launch_overlap.store(on ? 1 : 0, std::memory_order_relaxed); }

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace tg

extern "C" {

const char* tg_error_string(int code) {
  switch (code) {
    case TG_OK: return "ok";
    case TG_ERR_INVALID_ARGUMENT: return "invalid argument";
    case TG_ERR_MISALIGNED: return "pointer or stride not 16-byte aligned";
    case TG_ERR_UNSUPPORTED_DEVICE: return "device is not compute capability 10.0 (B200)";
    case TG_ERR_WORKSPACE: return "workspace missing or too small";
    case TG_ERR_CUDA: return "CUDA runtime or driver call failed";
    case TG_ERR_UNSUPPORTED_SHAPE: return "shape not implemented by the kernels";
    case TG_ERR_SCRATCH_LIMIT:
      return "size exceeds the fixed scratch of tg_gate_score_noalloc "
             "(TG_NOALLOC_MAX_TOKENS / TG_NOALLOC_MAX_HIDDEN)";
    default: return "unknown error";
  }
}

int tg_last_cuda_error(void) { return tg::g_last_cuda_error; }

int tg_device_supported(int device) {
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, device) != cudaSuccess)
    return 0;
  if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, device) != cudaSuccess)
    return 0;
  return (major == 10 && minor == 0) ? 1 : 0;
}

int tg_version(void) { return 100; }

int tg_plan_kept(const int32_t* cu_seqlens_host, const int32_t* n_question_host,
                 const int32_t* budgets_host, int batch, int32_t* cu_kept_host) {
  if (batch < 0 || !cu_kept_host) return TG_ERR_INVALID_ARGUMENT;
  if (batch > 0 && (!cu_seqlens_host || !n_question_host || !budgets_host))
    return TG_ERR_INVALID_ARGUMENT;
  if (batch > 0 && cu_seqlens_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  int64_t acc = 0;
  cu_kept_host[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    const int64_t q = n_question_host[b];
    if (n < 0 || q < 0 || q > n) return TG_ERR_INVALID_ARGUMENT;
    const int64_t d = n - q;
    int64_t kd = (int64_t)budgets_host[b] - q;
    if (kd < 0) kd = 0;
    if (kd > d) kd = d;
    acc += q + kd;
    if (acc > INT32_MAX) return TG_ERR_INVALID_ARGUMENT;
    cu_kept_host[b + 1] = (int32_t)acc;
  }
  return TG_OK;
}

int tg_set_launch_overlap(int enable) {
  tg::set_launch_overlap(enable != 0);
  return TG_OK;
}

int tg_get_launch_overlap(void) { return tg::launch_overlap() ? 1 : 0; }

int tg_set_gather_tma(int enable) {
  tg::g_gather_tma.store(enable ? 1 : 0);
  return TG_OK;
}

int tg_get_gather_tma(void) { return tg::gather_use_tma() ? 1 : 0; }

int tg_set_scorer_pair(int enable) {
  tg::g_scorer_pair.store(enable ? 1 : 0);
  return TG_OK;
}

int tg_get_scorer_pair(void) { return tg::scorer_use_pair() ? 1 : 0; }

int tg_status_clear(uint32_t* status, tg_stream_t stream) {
  if (!status) return TG_ERR_INVALID_ARGUMENT;
  TG_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(uint32_t), (cudaStream_t)stream));
  return TG_OK;
}

int tg_status_read(const uint32_t* status, uint32_t* out_host, tg_stream_t stream) {
  if (!status || !out_host) return TG_ERR_INVALID_ARGUMENT;
  TG_CUDA_TRY(cudaMemcpyAsync(out_host, status, sizeof(uint32_t), cudaMemcpyDeviceToHost,
                              (cudaStream_t)stream));
  TG_CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  return TG_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ L2 prefetch

namespace tg {
namespace {

constexpr uint32_t kPrefetchChunk = 32768;

// One thread per 32 KB chunk: a bulk L2 prefetch (a hint with no completion to wait for).
__global__ void prefetch_l2_kernel(const unsigned char* base, uint64_t bytes) {
  const uint64_t chunk = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const uint64_t off = chunk * kPrefetchChunk;
  if (off >= bytes) return;
  const uint64_t left = bytes - off;
  const uint32_t n = left < kPrefetchChunk ? (uint32_t)left : kPrefetchChunk;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                   reinterpret_cast<uint64_t>(base + off)),
               "r"(n)
               : "memory");
}

}  // namespace
}  // namespace tg

extern "C" int tg_prefetch_l2(const void* ptr, size_t bytes, tg_stream_t stream) {
  using namespace tg;
  if (bytes == 0) return TG_OK;
  if (!ptr) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(ptr)) return TG_ERR_MISALIGNED;
  const uint64_t n = (uint64_t)bytes & ~uint64_t(15);  // the bulk unit is 16 bytes
  if (n == 0) return TG_OK;
  TG_TRY(check_device());
  const uint64_t chunks = (n + kPrefetchChunk - 1) / kPrefetchChunk;
  const uint64_t blocks = (chunks + 127) / 128;
  if (blocks > 0x7FFFFFFFull) return TG_ERR_UNSUPPORTED_SHAPE;
  prefetch_l2_kernel<<<(unsigned)blocks, 128, 0, (cudaStream_t)stream>>>(
      static_cast<const unsigned char*>(ptr), n);
  return check_launch();
}
