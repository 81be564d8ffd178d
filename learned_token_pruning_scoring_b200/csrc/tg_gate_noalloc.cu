// Gate scoring for callers that cannot allocate device memory.
//
// Some callers of this library may not call cudaMalloc at all: a serving engine that
// plans every byte of device memory up front and forbids allocation while a request
// is in flight, a plug-in that only sees the buffers its host framework hands it, or
// a latency-critical path where cudaMalloc's implicit device synchronisation is not
// acceptable.  tg_gate_score needs a scratch workspace (the RMSNorm weight folded into
// W1 and per-32-row partial sums of s^2); this entry point takes it instead from a
// fixed array compiled into the library, so the caller passes only inputs and outputs.
//
// The array is a file-scope __device__ variable: every GPU that loads the library
// holds its kNoallocScratchBytes until the process exits.  Host code cannot use the
// array's name as a device address (it is a host-side stand-in), so the device address
// is looked up with cudaGetSymbolAddress once per device, on that device's first call.
#include <mutex>

#include "tg_host.h"

namespace tg {
namespace {

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Workspace layout of tg_gate_score at the largest supported shape.
constexpr size_t kNoallocScratchBytes =
    align256((size_t)256 * TG_NOALLOC_MAX_HIDDEN * 2) +
    align256((size_t)((TG_NOALLOC_MAX_TOKENS + 31) / 32 + 1) * sizeof(float));

static __device__ __align__(256) unsigned char g_gate_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_gate_scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return TG_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mutex);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    TG_CUDA_TRY(cudaGetSymbolAddress(&p, g_gate_scratch));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TG_OK;
}

}  // namespace
}  // namespace tg

extern "C" int tg_gate_score_noalloc(const tg_bf16* h, int64_t ld_h, int64_t total_tokens,
                                     int hidden, const float* norm_w, const tg_bf16* W1,
                                     int width, const float* w2, float eps_norm,
                                     const int32_t* cu_seqlens, const int32_t* cu_seqlens_host,
                                     int batch, float eps_seq, const uint8_t* prunable,
                                     float* s_out, float* z_out, float* bias_out,
                                     uint32_t* status, tg_stream_t stream) {
  // shapes tg_gate_score rejects get its error code, not the scratch limit
  if (width != 256 || hidden <= 0 || (hidden % 64)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (total_tokens > TG_NOALLOC_MAX_TOKENS || hidden > TG_NOALLOC_MAX_HIDDEN)
    return TG_ERR_SCRATCH_LIMIT;
  const size_t need = tg_gate_score_workspace_size(total_tokens, hidden, width, batch);
  if (need > tg::kNoallocScratchBytes) return TG_ERR_SCRATCH_LIMIT;
  TG_TRY(tg::check_device());
  void* scratch = nullptr;
  TG_TRY(tg::scratch_address(&scratch));
  // Nothing in the scratch has to start at zero: the folded weight is written before
  // the GEMM reads it, and every partial-sum slot the normalisation reads is written
  // by the scorer earlier in the same call.
  return tg_gate_score(h, ld_h, total_tokens, hidden, norm_w, W1, width, w2, eps_norm,
                       cu_seqlens, cu_seqlens_host, batch, eps_seq, prunable, s_out, z_out,
                       bias_out, scratch, tg::kNoallocScratchBytes, status, stream);
}
