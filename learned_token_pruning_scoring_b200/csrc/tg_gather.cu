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

// Per-row rotation table: the (cos, sin) row of each row's position, transposed so that
// block j (rotation pairs 2j, 2j + 1) of consecutive rows is contiguous:
// rot[j * ld_rot + r] = table[pos[r]][j] (float4).  One thread per (j, r), r fastest:
// the stores are coalesced, the table reads are gathers (once per step, not per layer).
__global__ void rope_rows_kernel(const int32_t* __restrict__ pos, int64_t n_rows,
                                 const float4* __restrict__ table, int max_pos, int blocks,
                                 float4* __restrict__ rot, int64_t ld_rot, uint32_t* status) {
  griddep_wait();
  const int64_t n = n_rows * blocks;
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int j = (int)(t / n_rows);
    const int64_t r = t % n_rows;
    int p = pos[r];
    if (p < 0 || p >= max_pos) {
      if (status) atomicOr(status, TG_STATUS_BOUNDS);
      p = 0;
    }
    rot[(int64_t)j * ld_rot + r] = table[(int64_t)p * blocks + j];
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

// ------------------------------------------------------------------ TMA row gather
//
// Gather mode through the tensor memory accelerator: groups of four kept rows come in
// with tile::gather4 loads (four row indices, box_cols columns per load, no swizzle) and
// leave with tiled TMA stores of four consecutive destination rows.  One CTA per SM
// walks a contiguous range of groups through a ring of stages (a stage is one group:
// width / box_cols chunks of 4 x box_cols elements, chunk j holding columns
// [j box_cols, (j + 1) box_cols) of the four rows).  Thread 0 issues the loads and the
// stores; a stage is refilled once its store has read it (bulk read groups) and, when
// row sums of squares are asked for, once the four warps (one per row) have read it.
// A group whose index is out of range loads row 0 in its place, stores only its valid
// rows (a one-row store map) and sets TG_STATUS_BOUNDS, as the copy kernel skips such
// rows; rows past n_rows of the last group are clipped by the store map.
constexpr int kTgThreads = 128;
constexpr int kTgMaxStages = 16;
constexpr int kTgSmemBudget = 192 * 1024;
constexpr int kTgRefillLag = 2;  // stores allowed to be still reading when a stage refills

struct TmaGatherArgs {
  const int32_t* row_idx;
  int64_t n_rows;
  int64_t src_rows;
  int width;
  int box_cols;
  int stages;
  int64_t n_groups;
  float* row_ssq;
  int64_t ld_ssq;
  uint32_t* status;
};

__global__ void __launch_bounds__(kTgThreads, 1)
    gather_tma_kernel(const __grid_constant__ CUtensorMap tm_src,
                      const __grid_constant__ CUtensorMap tm_dst4,
                      const __grid_constant__ CUtensorMap tm_dst1, TmaGatherArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int stage_bytes = 4 * a.width * 2;
  unsigned char* ring = smem_raw;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + a.stages * stage_bytes);
  uint32_t* valid = reinterpret_cast<uint32_t*>(full + kTgMaxStages);  // [stage] rows to store
  uint32_t* bad = valid + kTgMaxStages;                               // [stage] an index was bad

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t g0 = a.n_groups * blockIdx.x / gridDim.x;
  const int64_t g1 = a.n_groups * (blockIdx.x + 1) / gridDim.x;
  const int n_my = (int)(g1 - g0);
  const int chunks = a.width / a.box_cols;
  const int chunk_bytes = 4 * a.box_cols * 2;

  if (tid == 0) {
    for (int s = 0; s < a.stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
  }
  if (tid == 0) {
    tma_prefetch_desc(&tm_src);
    tma_prefetch_desc(&tm_dst4);
  }
  __syncthreads();
  griddep_wait();  // the indices and the source rows may come from the grid before

  auto issue = [&](int li) {  // thread 0: load group g0 + li into stage li % stages
    const int s = li % a.stages;
    const int64_t row0 = (g0 + li) * 4;
    int32_t r[4];
    uint32_t ok = 0, err = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t row = row0 + e;
      int64_t idx = 0;
      if (row < a.n_rows) {
        idx = a.row_idx ? (int64_t)a.row_idx[row] : row;
        if (idx < 0 || idx >= a.src_rows) {
          err = 1;
          idx = 0;
        } else {
          ok |= 1u << e;
        }
      }
      r[e] = (int32_t)idx;
    }
    if (err && a.status) atomicOr(a.status, TG_STATUS_BOUNDS);
    valid[s] = ok;
    bad[s] = err;
    unsigned char* st = ring + s * stage_bytes;
    mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
    for (int j = 0; j < chunks; ++j)
      tma_gather4(st + j * chunk_bytes, &tm_src, j * a.box_cols, r[0], r[1], r[2], r[3],
                  &full[s]);
  };
  auto store = [&](int li) {  // thread 0: store group g0 + li from its stage
    const int s = li % a.stages;
    const int64_t row0 = (g0 + li) * 4;
    const unsigned char* st = ring + s * stage_bytes;
    if (!bad[s]) {
      for (int j = 0; j < chunks; ++j)
        tma_store_2d(&tm_dst4, j * a.box_cols, (int32_t)row0, st + j * chunk_bytes);
    } else {
      for (int e = 0; e < 4; ++e)
        if (valid[s] >> e & 1u)
          for (int j = 0; j < chunks; ++j)
            tma_store_2d(&tm_dst1, j * a.box_cols, (int32_t)(row0 + e),
                         st + j * chunk_bytes + e * a.box_cols * 2);
    }
    bulk_commit_group();
  };

  const bool ssq = a.row_ssq != nullptr;
  if (tid == 0)
    for (int li = 0; li < n_my && li < a.stages; ++li) issue(li);
  if (ssq || tid == 0) {
    const int nvec = a.width >> 3;
    for (int li = 0; li < n_my; ++li) {
      const int s = li % a.stages;
      const uint32_t ph = (uint32_t)(li / a.stages) & 1u;
      bool ok = mbar_wait(&full[s], ph, nullptr, a.status);
      if (ssq) ok = __syncthreads_and(ok) != 0;
      if (!ok) break;  // a load that never landed (status has TIMEOUT): give up
      if (ssq) {
        // warp w: row w of the group; lane l sums vectors l, l + 32, ... (16 vectors =
        // one 128-column group, so each half-warp holds one group per step)
        const int64_t row = (g0 + li) * 4 + warp;
        const bool mine = (valid[s] >> warp & 1u) != 0;
        const unsigned char* st = ring + s * stage_bytes;
        for (int base = 0; base < nvec; base += 32) {
          const int v = base + lane;
          float q = 0.f;
          if (mine && v < nvec) {
            const int col = v * 8;
            const int j = col / a.box_cols;
            q = ssq8(*reinterpret_cast<const uint4*>(st + j * chunk_bytes +
                                                     (warp * a.box_cols + col - j * a.box_cols) * 2));
          }
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
          if (mine && v < nvec && (lane & 15) == 0) a.row_ssq[row * a.ld_ssq + (v >> 4)] = q;
        }
        fence_proxy_async_smem();  // these reads before the refill's TMA write
        __syncthreads();
      }
      if (tid == 0) {
        store(li);
        // refill the stage whose store is now at least kTgRefillLag groups old
        const int lr = li - kTgRefillLag;
        if (lr >= 0 && lr + a.stages < n_my) {
          bulk_wait_read<kTgRefillLag>();
          issue(lr + a.stages);
        }
      }
    }
    // the last kTgRefillLag stages were never refilled; nothing is left in flight but
    // stores, which must finish before the CTA exits
    if (tid == 0) bulk_wait_all();
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

// The TMA row gather for one call of the gather mode (width a multiple of 64).
int gather_tma(const GatherArgs& g, cudaStream_t stream) {
  const int box = (g.width % 256) == 0 ? 256 : (g.width % 128) == 0 ? 128 : 64;
  const int stage_bytes = 4 * g.width * 2;
  int stages = kTgSmemBudget / stage_bytes;
  if (stages > kTgMaxStages) stages = kTgMaxStages;
  const int64_t n_groups = (g.n_rows + 3) / 4;
  CUtensorMap ts, t4, t1;
  TG_TRY(make_tmap_bf16_2d_swz(&ts, g.src, (uint64_t)g.src_rows, (uint64_t)g.width,
                               (uint64_t)g.ld_src, (uint32_t)box, 1, false));
  TG_TRY(make_tmap_bf16_2d_swz(&t4, g.dst, (uint64_t)g.n_rows, (uint64_t)g.width,
                               (uint64_t)g.ld_dst, (uint32_t)box, 4, false));
  TG_TRY(make_tmap_bf16_2d_swz(&t1, g.dst, (uint64_t)g.n_rows, (uint64_t)g.width,
                               (uint64_t)g.ld_dst, (uint32_t)box, 1, false));
  const size_t smem = (size_t)stages * stage_bytes + kTgMaxStages * (8 + 4 + 4);
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(gather_tma_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kTgSmemBudget + kTgMaxStages * 16));
    attr_dev = dev;
  }
  TmaGatherArgs a{g.row_idx, g.n_rows, g.src_rows, g.width, box, stages, n_groups,
                  g.row_ssq, g.ld_ssq, g.status};
  const int64_t ctas = n_groups < sm_count() ? n_groups : sm_count();
  return launch(gather_tma_kernel, dim3((unsigned)ctas), dim3(kTgThreads), smem, stream, ts, t4,
                t1, a);
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

extern "C" int tg_rope_rows(const int32_t* pos, int64_t n_rows, const float* cos_sin,
                            int max_pos, int head_dim, float* rot, int64_t ld_rot,
                            uint32_t* status, tg_stream_t stream) {
  if (n_rows < 0 || max_pos <= 0 || ld_rot < n_rows) return TG_ERR_INVALID_ARGUMENT;
  if (head_dim < 8 || (head_dim & 3)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (n_rows == 0) return TG_OK;
  if (!pos || !cos_sin || !rot) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(cos_sin) || !aligned16(rot)) return TG_ERR_MISALIGNED;
  TG_TRY(check_device());
  const int blocks = head_dim / 4;
  const int64_t n = n_rows * blocks;
  int grid = (int)((n + 255) / 256);
  if (grid > sm_count() * 16) grid = sm_count() * 16;
  return launch(rope_rows_kernel, dim3(grid), dim3(256), 0, (cudaStream_t)stream, pos, n_rows,
                reinterpret_cast<const float4*>(cos_sin), max_pos, blocks,
                reinterpret_cast<float4*>(rot), ld_rot, status);
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
  if (!rope_pos || rope_col_begin >= rope_col_end) {
    if (gather_use_tma() && (width % 64) == 0 && width * 8 * (kTgRefillLag + 1) <= kTgSmemBudget &&
        src_rows < (int64_t)0x7FFFFFFF && n_rows < (int64_t)0x7FFFFFFF)
      return gather_tma(a, (cudaStream_t)stream);
    return launch(gather_copy_kernel, dim3(copy_grid(n_rows, kCopyBlocksPerSm)),
                  dim3(kCopyWarps * 32), 0, (cudaStream_t)stream, a);
  }
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
