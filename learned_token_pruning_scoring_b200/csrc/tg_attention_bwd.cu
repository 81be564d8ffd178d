// Backward of token-gated attention with respect to the gate: the key bias, the per-head
// gains and the temperature scale, on tcgen05 tensor cores.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 端到端训练的关键在 token 门控注意力 (the gate is trained end to end through the attention
// it biases); "TokenGate: Adapting LLMs for Fast and Memory-Efficient Prefill with
// Learned Token Pruning" (paper digest), 方法关键点.  With
//   l[r, c] = tau_r q_r.k_c / sqrt(d) + gamma_h b_c,  P = softmax_c(l),  O_r = sum_c P v_c
// and dO given, the softmax Jacobian gives dl[r, c] = P[r, c] (dO_r.v_c - dO_r.O_r), and
//   d_bias[c]  = sum_h gamma_h sum_r dl[r, c]
//   d_gamma[h] = sum_{r,c} dl[r, c] b_c
//   d_beta     = sum_h sum_{r,c} dl[r, c] (tau_r / beta) q_r.k_c / sqrt(d).
//
// Key-tile-major: one CTA = one request, one tile of 128 keys, one chunk of the query
// tiles at or after it, one kv head and the two q heads that read it.  Each thread of a
// head's four compute warps owns one key, so the sums over queries stay in its registers.
// Per query tile and head the tensor core computes, keys along M:
//   S^T  = K Q^T (+ one K=16 step adding g_r b_c, as in the forward)  -> TMEM [0,128)/[128,256)
//   dP^T = V dO^T                                                     -> TMEM [256,384)/[384,512)
// and the compute warps form P = 2^(t_r S - lse2_r) from the forward's log-sum-exp, then
// dl = P (dP - delta_r).  A preparation kernel lays out, per q head and query tile, one
// contiguous block: the gain operand of the bias step and the per-query scalars (t_r,
// lse2_r, delta_r = dO_r.O_r, and the temperature-gradient factors), with lse2 = +inf
// on rows past the request so that they contribute nothing; one bulk copy brings it in.
// Q and dO stages are freed by the MMAs that read them (so the next tile's loads overlap
// the compute warps), the blocks by the compute warps through a deeper ring.  Partial
// sums per (work item, head, key) go to the workspace and two small kernels reduce them
// in a fixed order (deterministic results).
// Warps: 0 producer (K, V and the key-bias operand once; per query tile and head Q and
// dO by TMA and the block by a bulk copy), 1 MMA issuer, 2-5 head h0, 6-9 head h0 + 1.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "tg_attn_common.cuh"
#include "tg_host.h"
#include "tg_ptx.cuh"

namespace tg {
namespace {

constexpr int kD = 128;       // head_dim
constexpr int kTq = 128;      // queries per tile
constexpr int kTk = 128;      // keys per tile
constexpr int kThreads = 320;
constexpr int kMaxBatch = 512;
constexpr int kTileBytes = 128 * kD * 2;  // 128 rows x 128 bf16 as two 64-column boxes
// Per (q head, query tile) block written by the preparation kernel: the gain operand
// (kAttnExBytes), float4 {t, lse2, delta, rho_s} per row, float u = rho_s g per row.
constexpr int kBlkGX = 0;
constexpr int kBlkA = kBlkGX + kAttnExBytes;
constexpr int kBlkU = kBlkA + kTq * 16;
constexpr int kBlockBytes = kBlkU + kTq * 4;
static_assert(kBlockBytes % 16 == 0, "bulk copies move multiples of 16 bytes");

// Work units u = 2 j + s: query tile j of the item, head s of the pair.  Q and dO stages
// follow the head (stage s), blocks a ring of four.
constexpr int kBlkStages = 4;
struct BwdSmem {
  static constexpr int K = 0;
  static constexpr int V = K + kTileBytes;
  static constexpr int Q = V + kTileBytes;               // [2]
  static constexpr int DO = Q + 2 * kTileBytes;          // [2]
  static constexpr int BLK = DO + 2 * kTileBytes;        // [kBlkStages]
  static constexpr int BX = BLK + kBlkStages * kBlockBytes;  // key-bias operand
  static constexpr int BAR = BX + kAttnExBytes;
  static constexpr int END = BAR + 256;
  static constexpr int BYTES = END + 1024;  // alignment slack
};
static_assert(BwdSmem::BYTES <= 227 * 1024, "shared memory budget");

struct BwdParams {
  const int32_t* cu_kept;
  const float* kept_bias;
  const unsigned char* blocks;  // [n_q_heads][n_tiles] blocks of kBlockBytes
  float* part;          // [item * head_groups + head group][2][2][128]
  int n_tiles;          // query tiles over all requests
  int group;            // n_q_heads / n_kv_heads
  int head_pairs;       // group / 2
  int n_kv_heads;
  int batch;
  int chunk;            // query tiles per work item
  uint32_t* status;
  int32_t item_prefix[kMaxBatch + 1];
  int32_t tile_prefix[kMaxBatch + 1];  // query (= key) tiles before request b
};

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// Work items of a request are (query chunk ci, key tile kt) in ci-major order, so that
// the CTAs running together read the same Q and dO tiles (L2 reuse).  Chunk ci covers
// query tiles [ci C, (ci + 1) C) and pairs with the key tiles kt < min(nt, (ci + 1) C);
// every chunk but the last is full, so the items before chunk ci number C ci (ci + 1) / 2.
constexpr int kMaxChunk = 16;  // query tiles per item at most (Q/dO working set in L2)
__host__ __device__ __forceinline__ int items_before_chunk(int ci, int C) {
  return C * ci * (ci + 1) / 2;
}
__host__ __device__ __forceinline__ int items_in_request(int nt, int C) {
  const int nch = (nt + C - 1) / C;
  return nch ? items_before_chunk(nch - 1, C) + nt : 0;
}

__device__ __forceinline__ int find_request(const int32_t* prefix, int batch, int t) {
  int lo = 0, hi = batch;  // largest b with prefix[b] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= t) lo = mid; else hi = mid;
  }
  return lo;
}

// ---------------------------------------------------------------- preparation
struct PrepParams {
  const uint16_t* o;
  int64_t ld_o;
  const uint16_t* d_o;
  int64_t ld_do;
  const float* lse;        // [n_q_heads, k_total], natural log
  const int32_t* cu_kept;
  const int32_t* kept_pos;
  const float* gamma;
  float beta;
  int n_q_heads;
  int64_t k_total;
  int batch;
  int n_tiles;
  unsigned char* blocks;
  int32_t tile_prefix[kMaxBatch + 1];
};

// Four threads per (q head, query tile, row of the tile): each loads a quarter of the
// row's dO and O (one batch of loads in flight), the quad sums delta, and its first
// thread writes the row's entries of the block.
__global__ void bwd_prep_kernel(const __grid_constant__ PrepParams p) {
  griddep_wait();
  const int64_t n = (int64_t)p.n_q_heads * p.n_tiles * kTq;
  const int quad = threadIdx.x & 3;
  const unsigned qmask = 0xFu << ((threadIdx.x & 31) & ~3u);
  for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 2; i < n;
       i += ((int64_t)gridDim.x * blockDim.x) >> 2) {
    const int rr = (int)(i % kTq);
    const int64_t ht = i / kTq;  // h * n_tiles + tile
    const int h = (int)(ht / p.n_tiles);
    const int tile = (int)(ht - (int64_t)h * p.n_tiles);
    const int b = find_request(p.tile_prefix, p.batch, tile);
    const int r = (tile - p.tile_prefix[b]) * kTq + rr;
    const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
    const bool valid = r < n_b;  // the same for the four threads
    const int64_t row = p.cu_kept[b] + r;
    float delta = 0.f;
    if (valid) {  // delta = dO_r . O_r over the head's 128 values, 32 per thread
      const uint4* x = reinterpret_cast<const uint4*>(p.d_o + row * p.ld_do + (int64_t)h * kD) +
                       quad * 4;
      const uint4* y = reinterpret_cast<const uint4*>(p.o + row * p.ld_o + (int64_t)h * kD) +
                       quad * 4;
      uint4 xv[4], yv[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        xv[k] = x[k];
        yv[k] = y[k];
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t xs[4] = {xv[k].x, xv[k].y, xv[k].z, xv[k].w};
        const uint32_t ys[4] = {yv[k].x, yv[k].y, yv[k].z, yv[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 fx = unpack_bf16x2(xs[e]), fy = unpack_bf16x2(ys[e]);
          delta = fmaf(fx.x, fy.x, delta);
          delta = fmaf(fx.y, fy.y, delta);
        }
      }
      delta += __shfl_xor_sync(qmask, delta, 1);
      delta += __shfl_xor_sync(qmask, delta, 2);
    }
    if (quad != 0) continue;
    unsigned char* blk = p.blocks + ht * kBlockBytes;
    float4 a = make_float4(0.f, INFINITY, 0.f, 0.f);
    float u = 0.f, g = 0.f;
    if (valid) {
      const int pos = p.kept_pos[row];
      const double tau = attn_tau(p.beta, r, pos);
      const float t = attn_logit_scale(tau, kD);
      g = p.gamma[h] * kAttnLog2e / t;
      // d l / d beta = (tau / beta) q.k / sqrt(d); tau / beta = 1 at pos = 0
      const double ratio = pos > 0 ? log((double)r + 1.0) / log((double)pos + 1.0) : 1.0;
      const float rho_s = (float)(ratio / sqrt((double)kD));
      a = make_float4(t, p.lse[(int64_t)h * p.k_total + row] * kAttnLog2e, delta, rho_s);
      u = rho_s * g;
    }
    attn_put_query_gain(blk + kBlkGX, rr, g);
    reinterpret_cast<float4*>(blk + kBlkA)[rr] = a;
    reinterpret_cast<float*>(blk + kBlkU)[rr] = u;
  }
}

// ---------------------------------------------------------------- main kernel
template <bool kBeta>
__global__ void __launch_bounds__(kThreads, 1)
    gated_attention_bias_grad_kernel(const __grid_constant__ CUtensorMap tmQ,
                                     const __grid_constant__ CUtensorMap tmK,
                                     const __grid_constant__ CUtensorMap tmV,
                                     const __grid_constant__ CUtensorMap tmDO,
                                     const __grid_constant__ BwdParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BwdSmem::BAR);
  uint64_t* kv_full = bars + 0;
  uint64_t* bx_full = bars + 1;
  uint64_t* q_full = bars + 2;       // [2]
  uint64_t* q_empty = bars + 4;      // [2] the S MMAs that read the stage are done
  uint64_t* do_full = bars + 6;      // [2]
  uint64_t* do_empty = bars + 8;     // [2] the dP MMAs that read the stage are done
  uint64_t* blk_full = bars + 10;    // [kBlkStages]
  uint64_t* blk_empty = bars + 14;   // [kBlkStages] MMAs + the head's 128 compute threads done
  uint64_t* s_full = bars + 18;      // [2] S^T and dP^T of the head in TMEM
  uint64_t* tmem_free = bars + 20;   // [2] the head's compute threads read them
  uint64_t* drain = bars + 22;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 23);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(kv_full, 1);
    mbar_init(bx_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&tmem_free[s], 128);
    }
    for (int s = 0; s < kBlkStages; ++s) {
      mbar_init(&blk_full[s], 1);
      mbar_init(&blk_empty[s], 1 + 128);  // the MMA commit + each compute thread
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmDO);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();

  // ---- work item: head groups vary fastest
  const int hg = p.n_kv_heads * p.head_pairs;
  const int head_grp = blockIdx.x % hg;
  const int item = blockIdx.x / hg;
  const int b = find_request(p.item_prefix, p.batch, item);
  const int64_t row0 = p.cu_kept[b];
  const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
  const int nt = cdiv(n_b, kTq);
  const int idx = item - p.item_prefix[b];
  int ci = 0;
  while (items_before_chunk(ci + 1, p.chunk) <= idx) ++ci;
  const int kt = idx - items_before_chunk(ci, p.chunk);
  const int qt_begin = max(kt, ci * p.chunk);
  const int nq = min(nt, (ci + 1) * p.chunk) - qt_begin;  // query tiles of this item (>= 1)
  const int g = head_grp / p.head_pairs;
  const int h0 = g * p.group + 2 * (head_grp % p.head_pairs);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const int ky = (int)(row0 + (int64_t)kt * kTk);
    if (lane == 0) {
      mbar_arrive_expect_tx(kv_full, 2 * kTileBytes);
      tma_load_2d(smem + BwdSmem::K, &tmK, g * kD, ky, kv_full);
      tma_load_2d(smem + BwdSmem::K + kTileBytes / 2, &tmK, g * kD + 64, ky, kv_full);
      tma_load_2d(smem + BwdSmem::V, &tmV, g * kD, ky, kv_full);
      tma_load_2d(smem + BwdSmem::V + kTileBytes / 2, &tmV, g * kD + 64, ky, kv_full);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int key = lane * 4 + e;
      const int c = kt * kTk + key;
      attn_put_key_bias(smem + BwdSmem::BX, key, c < n_b ? p.kept_bias[row0 + c] : 0.f);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bx_full);
    int n_q = 0, n_do = 0, n_blk = 0;  // loads issued into each ring
    for (int u = 0; u < 2 * nq; ++u) {
      const int s = u & 1;  // Q / dO stage = head of the pair
      const int bs = u % kBlkStages;
      const uint32_t ph2 = (uint32_t)(u >> 1) & 1u, ph4 = (uint32_t)(u / kBlkStages) & 1u;
      const int qt = qt_begin + (u >> 1);
      const int qy = (int)(row0 + (int64_t)qt * kTq);
      const int hh = h0 + s;
      if (!warp_all(mbar_wait(&q_empty[s], ph2 ^ 1u, abort_flag, p.status))) break;
      unsigned char* qs = smem + BwdSmem::Q + s * kTileBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[s], kTileBytes);
        tma_load_2d(qs, &tmQ, hh * kD, qy, &q_full[s]);
        tma_load_2d(qs + kTileBytes / 2, &tmQ, hh * kD + 64, qy, &q_full[s]);
      }
      ++n_q;
      if (!warp_all(mbar_wait(&blk_empty[bs], ph4 ^ 1u, abort_flag, p.status))) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&blk_full[bs], kBlockBytes);
        const int64_t blk = (int64_t)hh * p.n_tiles + p.tile_prefix[b] + qt;
        bulk_load(smem + BwdSmem::BLK + bs * kBlockBytes, p.blocks + blk * kBlockBytes,
                  kBlockBytes, &blk_full[bs]);
      }
      ++n_blk;
      if (!warp_all(mbar_wait(&do_empty[s], ph2 ^ 1u, abort_flag, p.status))) break;
      unsigned char* ds = smem + BwdSmem::DO + s * kTileBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&do_full[s], kTileBytes);
        tma_load_2d(ds, &tmDO, hh * kD, qy, &do_full[s]);
        tma_load_2d(ds + kTileBytes / 2, &tmDO, hh * kD + 64, qy, &do_full[s]);
      }
      ++n_do;
    }
    if (lane == 0) {
      // no bulk copy may still be landing when the CTA exits
      mbar_wait(kv_full, 0, nullptr, p.status);
      for (int u = n_q - 2 < 0 ? 0 : n_q - 2; u < n_q; ++u)
        mbar_wait(&q_full[u & 1], (uint32_t)(u >> 1) & 1u, nullptr, p.status);
      for (int u = n_do - 2 < 0 ? 0 : n_do - 2; u < n_do; ++u)
        mbar_wait(&do_full[u & 1], (uint32_t)(u >> 1) & 1u, nullptr, p.status);
      for (int u = n_blk - kBlkStages < 0 ? 0 : n_blk - kBlkStages; u < n_blk; ++u)
        mbar_wait(&blk_full[u % kBlkStages], (uint32_t)(u / kBlkStages) & 1u, nullptr,
                  p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false, false);
      const uint64_t k_desc = sw128_desc(smem_u32(smem + BwdSmem::K), 16, 1024);
      const uint64_t v_desc = sw128_desc(smem_u32(smem + BwdSmem::V), 16, 1024);
      const uint64_t bx_desc = interleave_desc(smem_u32(smem + BwdSmem::BX), 128, 256);
      bool ok = mbar_wait(kv_full, 0, abort_flag, p.status) &&
                mbar_wait(bx_full, 0, abort_flag, p.status);
      for (int u = 0; ok && u < 2 * nq; ++u) {
        const int s = u & 1;
        const int j = u >> 1;
        const int bs = u % kBlkStages;
        const uint32_t ph2 = (uint32_t)j & 1u, ph4 = (uint32_t)(u / kBlkStages) & 1u;
        if (!(ok = mbar_wait(&q_full[s], ph2, abort_flag, p.status) &&
                   mbar_wait(&blk_full[bs], ph4, abort_flag, p.status)))
          break;
        if (j > 0 && !(ok = mbar_wait(&tmem_free[s], (uint32_t)(j - 1) & 1u, abort_flag, p.status)))
          break;
        tc_fence_after();
        const uint32_t qs = smem_u32(smem + BwdSmem::Q + s * kTileBytes);
        const uint32_t ds = smem_u32(smem + BwdSmem::DO + s * kTileBytes);
        const uint64_t q_desc = sw128_desc(qs, 16, 1024);
        const uint64_t do_desc = sw128_desc(ds, 16, 1024);
        const uint64_t gx_desc =
            interleave_desc(smem_u32(smem + BwdSmem::BLK + bs * kBlockBytes + kBlkGX), 128, 256);
        const uint32_t s_col = tmem + (uint32_t)(s * 128);
        const uint32_t d_col = tmem + 256u + (uint32_t)(s * 128);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4);
          mma_ss(s_col, k_desc + off, q_desc + off, idesc, kk != 0);
        }
        mma_ss(s_col, bx_desc, gx_desc, idesc, 1u);  // + g_r b_c
        mma_commit(&q_empty[s]);
        if (!(ok = mbar_wait(&do_full[s], ph2, abort_flag, p.status))) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4);
          mma_ss(d_col, v_desc + off, do_desc + off, idesc, kk != 0);
        }
        mma_commit(&do_empty[s]);
        mma_commit(&s_full[s]);
        mma_commit(&blk_empty[bs]);
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.status);  // every MMA retired before TMEM is freed
    }
  } else {
    // ------------------------------------------------------------ per-key sums
    const int wg = (warp - 2) >> 2;  // 0: head h0, 1: head h0 + 1
    const int q = warp & 3;          // TMEM lane quarter this warp may access
    const int key = q * 32 + lane;
    const int c = kt * kTk + key;
    const float b_c = c < n_b ? p.kept_bias[row0 + c] : 0.f;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_t = tmem + lane_off + (uint32_t)(wg * 128);
    const uint32_t d_t = tmem + lane_off + 256u + (uint32_t)(wg * 128);
    float acc = 0.f, accb = 0.f;
    for (int j = 0; j < nq; ++j) {
      if (!warp_all(mbar_wait(&s_full[wg], (uint32_t)j & 1u, abort_flag, p.status))) break;
      tc_fence_after();
      const int bs = (2 * j + wg) % kBlkStages;
      // the block's bulk copy has landed (already true: the MMAs waited for it); waiting
      // on its barrier makes the copied scalars visible to this thread
      if (!warp_all(mbar_wait(&blk_full[bs], (uint32_t)((2 * j + wg) / kBlkStages) & 1u,
                              abort_flag, p.status)))
        break;
      const unsigned char* blk = smem + BwdSmem::BLK + bs * kBlockBytes;
      const float4* ca = reinterpret_cast<const float4*>(blk + kBlkA);
      const float* cu = reinterpret_cast<const float*>(blk + kBlkU);
      const bool diag = qt_begin + j == kt;  // queries before this key are masked
#pragma unroll 1
      for (int cc = 0; cc < kTq / 32; ++cc) {
        uint32_t sv[32], dv[32];
        tmem_ld32(s_t + 32 * cc, sv);
        tmem_ld32(d_t + 32 * cc, dv);
        tmem_wait_ld();
        if (cc == kTq / 32 - 1) {
          tc_fence_before();
          mbar_arrive(&tmem_free[wg]);  // the MMA may overwrite this head's S^T, dP^T
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int col = 32 * cc + i;
          const float4 a = ca[col];
          const float s = __uint_as_float(sv[i]);
          float pr = ex2_approx(fmaf(s, a.x, -a.y));
          if (diag && col < key) pr = 0.f;
          const float dl = pr * (__uint_as_float(dv[i]) - a.z);
          acc += dl;
          if (kBeta) accb = fmaf(dl, fmaf(a.w, s, -cu[col] * b_c), accb);
        }
      }
      // done with the block's scalars: every reading thread releases it itself, its
      // reads ordered (release, proxy fence) before the bulk copy that refills it
      fence_proxy_async_smem();
      mbar_arrive(&blk_empty[bs]);
    }
    const int64_t slot = (int64_t)item * hg + head_grp;
    p.part[((slot * 2 + 0) * 2 + wg) * 128 + key] = acc;
    p.part[((slot * 2 + 1) * 2 + wg) * 128 + key] = accb;
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- reductions
struct ReduceParams {
  const int32_t* cu_kept;
  const float* kept_bias;
  const float* gamma;
  const float* part;
  float* d_bias;
  float* tile_out;  // [tile][n_q_heads + 1]
  int n_q_heads;
  int group;
  int head_pairs;
  int n_kv_heads;
  int batch;
  int chunk;
  int32_t item_prefix[kMaxBatch + 1];
  int32_t tile_prefix[kMaxBatch + 1];
};

// One block per key tile, threads (key, head group): each thread sums its key's partials
// of the two heads of its group over the tile's items (all these loads are independent),
// then the block forms d_bias of its keys and, per head, the tile's sum of b_c * (sum
// over queries of dl), plus the tile's d_beta share, all in a fixed order.
constexpr int kReduceGroups = 8;  // blockDim.y
__global__ void __launch_bounds__(128 * kReduceGroups)
    bias_grad_reduce_kernel(const __grid_constant__ ReduceParams p) {
  extern __shared__ float red[];  // [n_q_heads][128] sums per head, [kReduceGroups][128] d_beta
  float* red_beta = red + p.n_q_heads * 128;
  griddep_wait();
  const int t = blockIdx.x;
  const int b = find_request(p.tile_prefix, p.batch, t);
  const int kt = t - p.tile_prefix[b];
  const int64_t row0 = p.cu_kept[b];
  const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
  const int n_chunks = cdiv(cdiv(n_b, kTq), p.chunk);
  const int hg = p.n_kv_heads * p.head_pairs;
  const int key = threadIdx.x;
  const int c = kt * kTk + key;
  const bool valid = c < n_b;
  float dbeta = 0.f;
  for (int grp = threadIdx.y; grp < hg; grp += kReduceGroups) {
    const int h0 = (grp / p.head_pairs) * p.group + 2 * (grp % p.head_pairs);
    float a0 = 0.f, a1 = 0.f;
    for (int ci = kt / p.chunk; ci < n_chunks; ++ci) {  // the items of this key tile
      const int item = p.item_prefix[b] + items_before_chunk(ci, p.chunk) + kt;
      const float* pp = p.part + ((int64_t)item * hg + grp) * 512 + key;
      a0 += pp[0];          // acc, head h0
      a1 += pp[128];        // acc, head h0 + 1
      dbeta += pp[256] + pp[384];
    }
    red[h0 * 128 + key] = a0;
    red[(h0 + 1) * 128 + key] = a1;
  }
  red_beta[threadIdx.y * 128 + key] = valid ? dbeta : 0.f;
  __syncthreads();
  if (threadIdx.y == 0) {
    const float b_c = valid ? p.kept_bias[row0 + c] : 0.f;
    float db = 0.f;
    for (int h = 0; h < p.n_q_heads; ++h) {
      const float a = red[h * 128 + key];
      db = fmaf(p.gamma[h], a, db);
      red[h * 128 + key] = valid ? b_c * a : 0.f;
    }
    if (valid) p.d_bias[row0 + c] = db;
  }
  __syncthreads();
  const int lin = threadIdx.y * 128 + threadIdx.x;
  for (int h = lin; h <= p.n_q_heads; h += 128 * kReduceGroups) {
    float sum = 0.f;
    if (h < p.n_q_heads) {
      for (int k = 0; k < 128; ++k) sum += red[h * 128 + k];
    } else {
      for (int y = 0; y < kReduceGroups; ++y)
        for (int k = 0; k < 128; ++k) sum += red_beta[y * 128 + k];
    }
    p.tile_out[(int64_t)t * (p.n_q_heads + 1) + h] = sum;
  }
}

__global__ void bias_grad_finish_kernel(const float* __restrict__ tile_out, int n_tiles,
                                        int n_q_heads, float* __restrict__ d_gamma,
                                        float* __restrict__ d_beta) {
  griddep_wait();
  for (int h = threadIdx.x; h <= n_q_heads; h += blockDim.x) {
    float sum = 0.f;
    for (int t = 0; t < n_tiles; ++t) sum += tile_out[(int64_t)t * (n_q_heads + 1) + h];
    if (h < n_q_heads) {
      if (d_gamma) d_gamma[h] = sum;
    } else if (d_beta) {
      *d_beta = sum;
    }
  }
}

// ---------------------------------------------------------------- host plan
struct BwdPlan {
  int chunk = 1;
  int n_items = 0;
  int n_tiles = 0;
};

// Query tiles per work item: the largest chunk (at most kMaxChunk) that still gives
// about two waves of CTAs.
int make_bwd_plan(const int32_t* cu_kept_host, int batch, int head_groups, int sms,
                  BwdPlan& plan, int32_t* item_prefix, int32_t* tile_prefix) {
  int max_nt = 1;
  tile_prefix[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int nt = cdiv(cu_kept_host[b + 1] - cu_kept_host[b], kTq);
    max_nt = std::max(max_nt, nt);
    tile_prefix[b + 1] = tile_prefix[b] + nt;
  }
  auto count = [&](int C) {
    int64_t items = 0;
    for (int b = 0; b < batch; ++b)
      items += items_in_request(cdiv(cu_kept_host[b + 1] - cu_kept_host[b], kTq), C);
    return items;
  };
  int C = std::min(max_nt, kMaxChunk);
  while (C > 1 && count(C) * head_groups < 2 * (int64_t)sms) --C;
  const int64_t items = count(C);
  if (items * head_groups > 0x7FFFFFFF) return TG_ERR_UNSUPPORTED_SHAPE;
  item_prefix[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int nt = cdiv(cu_kept_host[b + 1] - cu_kept_host[b], kTq);
    item_prefix[b + 1] = item_prefix[b] + items_in_request(nt, C);
  }
  plan.chunk = C;
  plan.n_items = (int)items;
  plan.n_tiles = tile_prefix[batch];
  return TG_OK;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct BwdLayout {
  size_t blocks, part, tile_out, total;
};

BwdLayout bwd_layout(int n_q_heads, int head_groups, const BwdPlan& plan) {
  BwdLayout l;
  l.blocks = 0;
  l.part = align256((size_t)n_q_heads * plan.n_tiles * kBlockBytes);
  l.tile_out = l.part + align256((size_t)plan.n_items * head_groups * 4 * 128 * sizeof(float));
  l.total = l.tile_out + align256((size_t)plan.n_tiles * (n_q_heads + 1) * sizeof(float));
  return l;
}

int validate(const int32_t* cu_kept_host, int batch, int n_q_heads, int n_kv_heads,
             int head_dim) {
  if (head_dim != kD) return TG_ERR_UNSUPPORTED_SHAPE;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads) return TG_ERR_INVALID_ARGUMENT;
  // the reduction keeps one 128-key row per q head in shared memory (<= 36 KB)
  if ((n_q_heads / n_kv_heads) % 2 || n_q_heads > 64) return TG_ERR_UNSUPPORTED_SHAPE;
  if (batch > kMaxBatch) return TG_ERR_UNSUPPORTED_SHAPE;
  if (batch < 0 || !cu_kept_host) return TG_ERR_INVALID_ARGUMENT;
  if (batch > 0 && cu_kept_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < batch; ++b)
    if (cu_kept_host[b + 1] < cu_kept_host[b]) return TG_ERR_INVALID_ARGUMENT;
  return TG_OK;
}

template <bool kBeta>
int set_bwd_smem() {
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(gated_attention_bias_grad_kernel<kBeta>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, BwdSmem::BYTES));
    attr_dev = dev;
  }
  return TG_OK;
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" size_t tg_gated_attention_bias_grad_workspace_size(const int32_t* cu_kept_host,
                                                              int batch, int n_q_heads,
                                                              int n_kv_heads, int head_dim) {
  if (validate(cu_kept_host, batch, n_q_heads, n_kv_heads, head_dim) != TG_OK || batch == 0)
    return 0;
  const int head_groups = n_q_heads / 2;
  BwdPlan plan;
  static thread_local int32_t ip[kMaxBatch + 1], tp[kMaxBatch + 1];
  if (make_bwd_plan(cu_kept_host, batch, head_groups, sm_count(), plan, ip, tp) != TG_OK)
    return 0;
  return bwd_layout(n_q_heads, head_groups, plan).total;
}

extern "C" int tg_gated_attention_bias_grad(
    const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k, const tg_bf16* v,
    int64_t ld_v, const tg_bf16* o, int64_t ld_o, const tg_bf16* d_o, int64_t ld_do,
    const float* lse, const int32_t* cu_kept, const int32_t* cu_kept_host, int batch,
    int n_q_heads, int n_kv_heads, int head_dim, const int32_t* kept_pos,
    const float* kept_bias, const float* gamma, float beta, float* d_bias, float* d_gamma,
    float* d_beta, void* workspace, size_t workspace_bytes, uint32_t* status,
    tg_stream_t stream) {
  TG_TRY(validate(cu_kept_host, batch, n_q_heads, n_kv_heads, head_dim));
  if (!std::isfinite(beta) || beta < 0.f) return TG_ERR_INVALID_ARGUMENT;
  const int64_t k_total = batch > 0 ? cu_kept_host[batch] : 0;
  if (k_total == 0 && !d_gamma && !d_beta) return TG_OK;
  if (k_total > 0) {
    if (!q || !k || !v || !o || !d_o || !lse || !cu_kept || !kept_pos || !kept_bias || !gamma ||
        !d_bias)
      return TG_ERR_INVALID_ARGUMENT;
    if (ld_q < (int64_t)n_q_heads * kD || ld_o < (int64_t)n_q_heads * kD ||
        ld_do < (int64_t)n_q_heads * kD || ld_k < (int64_t)n_kv_heads * kD ||
        ld_v < (int64_t)n_kv_heads * kD)
      return TG_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(d_o) ||
        !stride_ok(ld_q, 2) || !stride_ok(ld_k, 2) || !stride_ok(ld_v, 2) ||
        !stride_ok(ld_o, 2) || !stride_ok(ld_do, 2))
      return TG_ERR_MISALIGNED;
  }
  TG_TRY(check_device());
  const int group = n_q_heads / n_kv_heads;
  const int head_groups = n_kv_heads * (group / 2);
  BwdPlan plan;
  ReduceParams rp{};
  TG_TRY(make_bwd_plan(cu_kept_host, batch, head_groups, sm_count(), plan, rp.item_prefix,
                       rp.tile_prefix));
  const BwdLayout lay = bwd_layout(n_q_heads, head_groups, plan);
  if (lay.total > 0 && (!workspace || workspace_bytes < lay.total)) return TG_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return TG_ERR_MISALIGNED;
  unsigned char* ws = static_cast<unsigned char*>(workspace);
  cudaStream_t st = (cudaStream_t)stream;
  float* tile_out = reinterpret_cast<float*>(ws + lay.tile_out);

  if (k_total > 0) {
    unsigned char* blocks = ws + lay.blocks;
    PrepParams pp{};
    pp.o = reinterpret_cast<const uint16_t*>(o);
    pp.ld_o = ld_o;
    pp.d_o = reinterpret_cast<const uint16_t*>(d_o);
    pp.ld_do = ld_do;
    pp.lse = lse;
    pp.cu_kept = cu_kept;
    pp.kept_pos = kept_pos;
    pp.gamma = gamma;
    pp.beta = beta;
    pp.n_q_heads = n_q_heads;
    pp.k_total = k_total;
    pp.batch = batch;
    pp.n_tiles = plan.n_tiles;
    pp.blocks = blocks;
    std::copy(rp.tile_prefix, rp.tile_prefix + kMaxBatch + 1, pp.tile_prefix);
    const int64_t n = (int64_t)n_q_heads * plan.n_tiles * kTq * 4;  // threads: four per row
    int64_t grid = (n + 255) / 256;
    if (grid > 16 * (int64_t)sm_count()) grid = 16 * (int64_t)sm_count();
    TG_TRY(launch(bwd_prep_kernel, dim3((unsigned)grid), dim3(256), 0, st, pp));

    CUtensorMap tq, tk, tv, tdo;
    TG_TRY(make_tmap_bf16_2d(&tq, q, (uint64_t)k_total, (uint64_t)n_q_heads * kD, (uint64_t)ld_q,
                             64, kTq));
    TG_TRY(make_tmap_bf16_2d(&tk, k, (uint64_t)k_total, (uint64_t)n_kv_heads * kD,
                             (uint64_t)ld_k, 64, kTk));
    TG_TRY(make_tmap_bf16_2d(&tv, v, (uint64_t)k_total, (uint64_t)n_kv_heads * kD,
                             (uint64_t)ld_v, 64, kTk));
    TG_TRY(make_tmap_bf16_2d(&tdo, d_o, (uint64_t)k_total, (uint64_t)n_q_heads * kD,
                             (uint64_t)ld_do, 64, kTq));
    BwdParams bp{};
    bp.cu_kept = cu_kept;
    bp.kept_bias = kept_bias;
    bp.blocks = blocks;
    bp.part = reinterpret_cast<float*>(ws + lay.part);
    bp.n_tiles = plan.n_tiles;
    bp.group = group;
    bp.head_pairs = group / 2;
    bp.n_kv_heads = n_kv_heads;
    bp.batch = batch;
    bp.chunk = plan.chunk;
    bp.status = status;
    std::copy(rp.item_prefix, rp.item_prefix + kMaxBatch + 1, bp.item_prefix);
    std::copy(rp.tile_prefix, rp.tile_prefix + kMaxBatch + 1, bp.tile_prefix);
    const int64_t cta = (int64_t)plan.n_items * head_groups;
    if (cta > 0) {
      if (d_beta) {
        TG_TRY(set_bwd_smem<true>());
        TG_TRY(launch(gated_attention_bias_grad_kernel<true>, dim3((unsigned)cta),
                      dim3(kThreads), BwdSmem::BYTES, st, tq, tk, tv, tdo, bp));
      } else {
        TG_TRY(set_bwd_smem<false>());
        TG_TRY(launch(gated_attention_bias_grad_kernel<false>, dim3((unsigned)cta),
                      dim3(kThreads), BwdSmem::BYTES, st, tq, tk, tv, tdo, bp));
      }
      rp.cu_kept = cu_kept;
      rp.kept_bias = kept_bias;
      rp.gamma = gamma;
      rp.part = bp.part;
      rp.d_bias = d_bias;
      rp.tile_out = tile_out;
      rp.n_q_heads = n_q_heads;
      rp.group = group;
      rp.head_pairs = group / 2;
      rp.n_kv_heads = n_kv_heads;
      rp.batch = batch;
      rp.chunk = plan.chunk;
      TG_TRY(launch(bias_grad_reduce_kernel, dim3((unsigned)plan.n_tiles),
                    dim3(128, kReduceGroups),
                    (size_t)(n_q_heads + kReduceGroups) * 128 * sizeof(float), st, rp));
    }
  }
  return launch(bias_grad_finish_kernel, dim3(1), dim3(std::min(1024, n_q_heads + 1)), 0, st,
                (const float*)tile_out, plan.n_tiles, n_q_heads, d_gamma, d_beta);
}
