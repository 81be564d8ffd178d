// Row gather with original-position RoPE, compacted KV-cache writes, and the rotary
// table.  These are HBM-bound copies: one warp moves one row with 16-byte accesses,
// all loads of a row issued before its stores, as many warps resident per SM as the
// kernel's registers allow.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 门控到底插在模型的哪个位置 (pruned rows stop at the gate; only kept rows go up);
// "TokenGate：让模型学会跳读，而不只压缩 KV 缓存", figure 1(a)(b) (kept tokens keep their
// original position encoding; upper layers store KV only for kept positions);
// "TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill with Learned Token
// Pruning" (paper digest), section 方法关键点 (the KV cache can be selectively trimmed).
#include <cuda_bf16.h>

#include <cstdint>

#include "tg_host.h"
#include "tg_ptx.cuh"

namespace tg {
namespace {

constexpr int kCopyWarps = 8;     // warps per block
constexpr int kVecPerBatch = 8;   // 16-byte vectors in flight per lane

__global__ void rope_table_kernel(float2* __restrict__ table, int max_pos, int half,
                                  double theta, int head_dim) {
  griddep_wait();
  const int64_t n = (int64_t)max_pos * half;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int p = (int)(t / half);
    const int i = (int)(t % half);
    const double inv_freq = pow(theta, -2.0 * (double)i / (double)head_dim);
    double s, c;
    sincos((double)p * inv_freq, &s, &c);
    table[t] = make_float2((float)c, (float)s);
  }
}

// Plain row copy of `nvec` 16-byte vectors (lane-strided), all loads before stores.
__device__ __forceinline__ void copy_row(const uint4* __restrict__ s, uint4* __restrict__ d,
                                         int vbegin, int vend, int lane) {
  for (int base = vbegin; base < vend; base += 32 * kVecPerBatch) {
    uint4 buf[kVecPerBatch];
#pragma unroll
    for (int u = 0; u < kVecPerBatch; ++u) {
      const int v = base + u * 32 + lane;
      if (v < vend) buf[u] = s[v];
    }
#pragma unroll
    for (int u = 0; u < kVecPerBatch; ++u) {
      const int v = base + u * 32 + lane;
      if (v < vend) d[v] = buf[u];
    }
  }
}

__device__ __forceinline__ void rotate8(uint4& a, uint4& b, const float4* __restrict__ cs) {
  // a: 8 elements of the first half, b: the matching 8 of the second half.
  uint32_t* pa = reinterpret_cast<uint32_t*>(&a);
  uint32_t* pb = reinterpret_cast<uint32_t*>(&b);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 t = cs[k];  // (cos_j, sin_j, cos_j+1, sin_j+1)
    const float2 x1 = unpack_bf16x2(pa[k]);
    const float2 x2 = unpack_bf16x2(pb[k]);
    const float y1a = x1.x * t.x - x2.x * t.y;
    const float y2a = x2.x * t.x + x1.x * t.y;
    const float y1b = x1.y * t.z - x2.y * t.w;
    const float y2b = x2.y * t.z + x1.y * t.w;
    pa[k] = pack_bf16x2(y1a, y1b);
    pb[k] = pack_bf16x2(y2a, y2b);
  }
}

struct GatherArgs {
  const uint16_t* src;
  int64_t ld_src;
  int64_t src_rows;
  const int32_t* row_idx;
  int64_t n_rows;
  int width;
  const int32_t* rope_pos;
  int rope_begin, rope_end, head_dim;
  const float* cos_sin;
  int max_pos;
  uint16_t* dst;
  int64_t ld_dst;
  float* row_ssq;  // optional: sums of squares of each gathered row per 128 columns
  int64_t ld_ssq;
  uint32_t* status;
};

// Sum of squares of the 8 bf16 values of one 16-byte vector.
__device__ __forceinline__ float ssq8(const uint4& v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = unpack_bf16x2(w[e]);
    s = fmaf(f.x, f.x, s);
    s = fmaf(f.y, f.y, s);
  }
  return s;
}

// Gathered copy of one row that also writes its sums of squares per 128 columns
// (16 vectors): lane l holds vectors l, l+32, ...; groups of 16 lanes share a group.
__device__ __forceinline__ void copy_row_ssq(const uint4* __restrict__ s, uint4* __restrict__ d,
                                             int nvec, int lane, float* ssq_row) {
  for (int base = 0; base < nvec; base += 32 * kVecPerBatch) {
    uint4 buf[kVecPerBatch];
#pragma unroll
    for (int u = 0; u < kVecPerBatch; ++u) {
      const int v = base + u * 32 + lane;
      if (v < nvec) buf[u] = s[v];
    }
#pragma unroll
    for (int u = 0; u < kVecPerBatch; ++u) {
      const int v = base + u * 32 + lane;
      float q = v < nvec ? ssq8(buf[u]) : 0.f;
      // reduce over the 16 lanes of this half-warp (vectors of one 128-column group)
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
      if (v < nvec) {
        d[v] = buf[u];
        if ((lane & 15) == 0) ssq_row[v >> 4] = q;
      }
    }
  }
}

// Plain gather (no RoPE): one warp per row, optional per-128-column sums of squares.
// Kept apart from the RoPE kernel so that its registers stay within 64 per thread and
// four blocks (32 warps, 4 KB in flight each) fit on every SM.
constexpr int kCopyBlocksPerSm = 4;
__global__ void __launch_bounds__(kCopyWarps * 32, kCopyBlocksPerSm)
    gather_copy_kernel(GatherArgs a) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kCopyWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kCopyWarps;
  const int nvec = a.width >> 3;
  for (int64_t r = warp0; r < a.n_rows; r += nwarps) {
    const int64_t sr = a.row_idx ? (int64_t)a.row_idx[r] : r;
    if (sr < 0 || sr >= a.src_rows) {
      if (lane == 0 && a.status) atomicOr(a.status, TG_STATUS_BOUNDS);
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(a.src + sr * a.ld_src);
    uint4* d = reinterpret_cast<uint4*>(a.dst + r * a.ld_dst);
    if (a.row_ssq) copy_row_ssq(s, d, nvec, lane, a.row_ssq + r * a.ld_ssq);
    else copy_row(s, d, 0, nvec, lane);
  }
}

__global__ void __launch_bounds__(kCopyWarps * 32) gather_rope_kernel(GatherArgs a) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kCopyWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kCopyWarps;
  const int nvec = a.width >> 3;
  for (int64_t r = warp0; r < a.n_rows; r += nwarps) {
    const int64_t sr = a.row_idx ? (int64_t)a.row_idx[r] : r;
    if (sr < 0 || sr >= a.src_rows) {
      if (lane == 0 && a.status) atomicOr(a.status, TG_STATUS_BOUNDS);
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(a.src + sr * a.ld_src);
    uint4* d = reinterpret_cast<uint4*>(a.dst + r * a.ld_dst);
    const int pos = a.rope_pos ? a.rope_pos[r] : -1;
    if (a.rope_pos && (pos < 0 || pos >= a.max_pos) && lane == 0 && a.status)
      atomicOr(a.status, TG_STATUS_BOUNDS);
    if (pos < 0 || pos >= a.max_pos || a.rope_begin >= a.rope_end) {
      if (a.row_ssq) copy_row_ssq(s, d, nvec, lane, a.row_ssq + r * a.ld_ssq);
      else copy_row(s, d, 0, nvec, lane);
      continue;
    }
    const int vb = a.rope_begin >> 3, ve = a.rope_end >> 3;
    copy_row(s, d, 0, vb, lane);
    copy_row(s, d, ve, nvec, lane);
    // Rotated span: tasks = (head, 8-element group of the first half).
    const int half = a.head_dim >> 1;
    const int groups = half >> 3;
    const int ntask = ((a.rope_end - a.rope_begin) / a.head_dim) * groups;
    const float4* cs_row = reinterpret_cast<const float4*>(a.cos_sin + (int64_t)pos * half * 2);
    for (int t = lane; t < ntask; t += 32) {
      const int hh = t / groups, g = t % groups;
      const int c1 = a.rope_begin + hh * a.head_dim + g * 8;
      uint4 x1 = s[c1 >> 3];
      uint4 x2 = s[(c1 + half) >> 3];
      rotate8(x1, x2, cs_row + g * 4);
      d[c1 >> 3] = x1;
      d[(c1 + half) >> 3] = x2;
    }
  }
}

struct KvArgs {
  const uint16_t* k;
  int64_t ld_k;
  const uint16_t* v;
  int64_t ld_v;
  int64_t src_rows;
  const int32_t* row_idx;
  int64_t n_rows;
  int width;
  uint16_t* ck;
  uint16_t* cv;
  int64_t ld_c;
  int64_t slot;
  uint32_t* status;
};

__global__ void __launch_bounds__(kCopyWarps * 32, kCopyBlocksPerSm) kv_compact_kernel(KvArgs a) {
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t warp0 = (int64_t)blockIdx.x * kCopyWarps + (threadIdx.x >> 5);
  const int64_t nwarps = (int64_t)gridDim.x * kCopyWarps;
  const int nvec = a.width >> 3;
  for (int64_t t = warp0; t < 2 * a.n_rows; t += nwarps) {
    const bool is_v = t >= a.n_rows;
    const int64_t r = is_v ? t - a.n_rows : t;
    const int64_t sr = a.row_idx ? (int64_t)a.row_idx[r] : r;
    if (sr < 0 || sr >= a.src_rows) {
      if (lane == 0 && a.status) atomicOr(a.status, TG_STATUS_BOUNDS);
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(is_v ? a.v + sr * a.ld_v : a.k + sr * a.ld_k);
    uint4* d = reinterpret_cast<uint4*>((is_v ? a.cv : a.ck) + (a.slot + r) * a.ld_c);
    copy_row(s, d, 0, nvec, lane);
  }
}

// One warp per row, at most the blocks that are resident at once (the kernels stride
// over the rest).
int copy_grid(int64_t rows, int blocks_per_sm) {
  const int64_t want = (rows + kCopyWarps - 1) / kCopyWarps;
  const int64_t cap = (int64_t)sm_count() * blocks_per_sm;
  return (int)(want < cap ? (want < 1 ? 1 : want) : cap);
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" int tg_rope_table(float* cos_sin, int max_pos, int head_dim, double theta,
                             tg_stream_t stream) {
  if (!cos_sin || max_pos <= 0 || head_dim <= 0 || (head_dim & 1) || !(theta > 1.0))
    return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  const int half = head_dim / 2;
  const int64_t n = (int64_t)max_pos * half;
  int grid = (int)((n + 255) / 256);
  if (grid > sm_count() * 16) grid = sm_count() * 16;
  return launch(rope_table_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream,
                reinterpret_cast<float2*>(cos_sin), max_pos, half, theta, head_dim);
}

extern "C" int tg_gather_rope(const tg_bf16* src, int64_t ld_src, int64_t src_rows,
                              const int32_t* row_idx, int64_t n_rows, int width,
                              const int32_t* rope_pos, int rope_col_begin, int rope_col_end,
                              int head_dim, const float* cos_sin, int max_pos, tg_bf16* dst,
                              int64_t ld_dst, float* row_ssq_out, int64_t ld_ssq_out,
                              uint32_t* status, tg_stream_t stream) {
  if (n_rows < 0 || width <= 0 || (width & 7) || src_rows < 0) return TG_ERR_INVALID_ARGUMENT;
  if (!row_idx && n_rows > src_rows) return TG_ERR_INVALID_ARGUMENT;
  if (n_rows == 0) return TG_OK;
  if (!src || !dst) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(src) || !aligned16(dst) || !stride_ok(ld_src, 2) || !stride_ok(ld_dst, 2))
    return TG_ERR_MISALIGNED;
  if (ld_src < width || ld_dst < width) return TG_ERR_INVALID_ARGUMENT;
  if (row_idx && src == dst) return TG_ERR_INVALID_ARGUMENT;
  if (row_ssq_out && (rope_pos || (width % 128) || ld_ssq_out < width / 128))
    return TG_ERR_INVALID_ARGUMENT;
  if (rope_pos) {
    if (!cos_sin || max_pos <= 0 || head_dim < 16 || (head_dim & 15)) return TG_ERR_INVALID_ARGUMENT;
    if (rope_col_begin < 0 || rope_col_end > width || rope_col_begin > rope_col_end ||
        rope_col_begin % head_dim || rope_col_end % head_dim)
      return TG_ERR_INVALID_ARGUMENT;
    if (!aligned16(cos_sin)) return TG_ERR_MISALIGNED;
  }
  TG_TRY(check_device());
  GatherArgs a{reinterpret_cast<const uint16_t*>(src), ld_src, src_rows, row_idx, n_rows, width,
               rope_pos, rope_col_begin, rope_col_end, head_dim, cos_sin, max_pos,
               reinterpret_cast<uint16_t*>(dst), ld_dst, row_ssq_out, ld_ssq_out, status};
  if (!rope_pos || rope_col_begin >= rope_col_end)
    return launch(gather_copy_kernel, dim3(copy_grid(n_rows, kCopyBlocksPerSm)),
                  dim3(kCopyWarps * 32), 0, (cudaStream_t)stream, a);
  // the RoPE kernel is register-heavy (one block per SM); it serves the unfused path
  return launch(gather_rope_kernel, dim3(copy_grid(n_rows, 1)), dim3(kCopyWarps * 32), 0,
                (cudaStream_t)stream, a);
}

extern "C" int tg_kv_compact(const tg_bf16* k, int64_t ld_k, const tg_bf16* v, int64_t ld_v,
                             int64_t src_rows, const int32_t* row_idx, int64_t n_rows, int width,
                             tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache,
                             int64_t cache_rows, int64_t slot_offset, uint32_t* status,
                             tg_stream_t stream) {
  if (n_rows < 0 || width <= 0 || (width & 7) || slot_offset < 0 || src_rows < 0)
    return TG_ERR_INVALID_ARGUMENT;
  if (slot_offset + n_rows > cache_rows) return TG_ERR_INVALID_ARGUMENT;
  if (!row_idx && n_rows > src_rows) return TG_ERR_INVALID_ARGUMENT;
  if (n_rows == 0) return TG_OK;
  if (!k || !v || !cache_k || !cache_v) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(k) || !aligned16(v) || !aligned16(cache_k) || !aligned16(cache_v) ||
      !stride_ok(ld_k, 2) || !stride_ok(ld_v, 2) || !stride_ok(ld_cache, 2))
    return TG_ERR_MISALIGNED;
  if (ld_k < width || ld_v < width || ld_cache < width) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  KvArgs a{reinterpret_cast<const uint16_t*>(k), ld_k, reinterpret_cast<const uint16_t*>(v), ld_v,
           src_rows, row_idx, n_rows, width, reinterpret_cast<uint16_t*>(cache_k),
           reinterpret_cast<uint16_t*>(cache_v), ld_cache, slot_offset, status};
  return launch(kv_compact_kernel, dim3(copy_grid(2 * n_rows, kCopyBlocksPerSm)),
                dim3(kCopyWarps * 32), 0, (cudaStream_t)stream, a);
}
