// Host-side helpers shared by the entry points: error bookkeeping, device checks,
// alignment checks and TMA tensor-map encoding (through the driver entry point, so
// the library needs no link-time dependency on libcuda).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "tokengate.h"

namespace tg {

void set_cuda_error(cudaError_t e);

// TG_ERR_UNSUPPORTED_DEVICE unless the current device is compute capability 10.0.
int check_device();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Row stride (elements) times element size must be a multiple of 16 bytes.
inline bool stride_ok(int64_t ld, int elem_bytes) { return ld > 0 && (ld * elem_bytes) % 16 == 0; }

// Returns TG_ERR_CUDA (and records the error) if the last launch failed.
int check_launch();

// 2-D bf16 row-major tensor [rows, cols] with row stride `ld` elements, tiled in boxes
// of box_cols x box_rows with 128-byte swizzle (box_cols * 2 must be 128).  Elements
// outside the tensor read as zero.
int make_tmap_bf16_2d(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                      uint64_t ld, uint32_t box_cols, uint32_t box_rows);

// The same with the swizzle chosen: swizzle128 = false lays a box out plainly, row after
// row (box_cols * 2 a multiple of 16, box_cols <= 256).
int make_tmap_bf16_2d_swz(CUtensorMap* out, const void* base, uint64_t rows, uint64_t cols,
                          uint64_t ld, uint32_t box_cols, uint32_t box_rows, bool swizzle128);

// Number of SMs of the current device (cached).
int sm_count();

// Library-wide switch (tg_set_launch_overlap): launch kernels with programmatic stream
// serialisation so that a grid's launch and prologue overlap the end of the grid before it.
bool launch_overlap();
// Library-wide switch (tg_set_gather_tma): the gather mode of tg_gather_rope uses the TMA
// row-gather kernel where the shape allows it, else (the default) the warp-per-row copy.
bool gather_use_tma();
// Library-wide switch (tg_set_scorer_pair): the scorer GEMM of tg_gate_score runs on CTA
// pairs (the default) or on one CTA per 128-row tile.
bool scorer_use_pair();
void set_launch_overlap(bool on);

// Launch `kernel` on `stream`, with programmatic stream serialisation when the switch is
// on.  Every kernel launched this way calls griddep_wait() before it touches global
// memory that an earlier grid may write.  Returns TG_OK or TG_ERR_CUDA.
template <typename... KArgs, typename... Args>
int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
           Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = launch_overlap() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return TG_ERR_CUDA;
  }
  return TG_OK;
}

}  // namespace tg

#define TG_CUDA_TRY(expr)                      \
  do {                                         \
    cudaError_t _e = (expr);                   \
    if (_e != cudaSuccess) {                   \
      ::tg::set_cuda_error(_e);                \
      return TG_ERR_CUDA;                      \
    }                                          \
  } while (0)

#define TG_TRY(expr)             \
  do {                           \
    int _rc = (expr);            \
    if (_rc != TG_OK) return _rc; \
  } while (0)
