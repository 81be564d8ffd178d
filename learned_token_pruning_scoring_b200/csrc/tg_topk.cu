// Prunable-only top-K selection with stable, order-preserving compaction.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 门控到底插在模型的哪个位置 (keep the top-K tokens by score; the question and other
// non-prunable tokens always take part); "斯坦福与 UC Berkeley 提出 TokenGate：token 门控注意力
// 让长上下文预填充最高快 11.3 倍", section "How does TokenGate learned token pruning work?"
// (only the document is prunable); "TokenGate：让模型学会跳读，而不只压缩 KV 缓存",
// figure 1(a)(b) (kept tokens keep their original positions).
//
// Design: one thread-block cluster of kCluster CTAs per request.  Each CTA owns a
// contiguous slice of the request, each warp a contiguous sub-slice.  Scores become
// order-preserving 32-bit keys (larger float -> larger key, -0 == +0, NaN lowest),
// cached in shared memory when the slice fits.  Three radix passes (11, 11, 10 bits)
// find the key T of the Kd-th best prunable token: per-CTA histograms (warp-aggregated
// shared atomics) are summed across the cluster through distributed shared memory.
// Ties at T go to the lowest indices.  A counting pass and a cluster exchange give
// every CTA and warp its output offset; the write pass compacts with warp ballots, so
// kept tokens come out in position order.  All counts are integers: the result is
// exact and deterministic.
#include <cooperative_groups.h>

#include <cstdint>

#include "tg_host.h"
#include "tg_ptx.cuh"
#include "tg_ptx.cuh"

namespace cg = cooperative_groups;

namespace tg {
namespace {

constexpr int kCluster = 8;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kSmemKeys = 16384;  // keys cached per CTA (slice up to this size)

struct TopkArgs {
  const float* z;
  const uint8_t* prunable;
  const int32_t* cu_seqlens;
  const int32_t* cu_kept;
  int32_t* kept_idx;
  int32_t* kept_pos;
  float* kept_bias;
  uint32_t* status;
};

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) return 0u;  // NaN: below every number
  if (u == 0x80000000u) u = 0u;                    // -0 == +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
  uint32_t hist[2][kBins];
  uint32_t tot[kBins];
  uint32_t xchg[4];             // values peers read: q, gt, eq counts of this CTA
  uint32_t warp_cnt[kWarps][3];  // q, gt, eq per warp
  uint32_t warp_sel_eq[kWarps];
  uint32_t warp_out[kWarps];
  uint32_t scan[kWarps];
  uint32_t sel_bin, count_above;
  uint32_t keys[kSmemKeys];
  uint8_t pr[kSmemKeys];
};

// Block-wide exclusive suffix sum of one value per thread: sum over threads with a
// higher index.
__device__ __forceinline__ uint32_t block_suffix_excl(uint32_t v, uint32_t* scan_smem) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // inclusive suffix within the warp
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_down_sync(0xFFFFFFFFu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) scan_smem[warp] = x;  // warp total
  __syncthreads();
  uint32_t after = 0;
  for (int w = warp + 1; w < kWarps; ++w) after += scan_smem[w];
  __syncthreads();
  return after + (x - v);
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kThreads)
    topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Shared& S = *reinterpret_cast<Shared*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int crank = (int)cluster.block_rank();
  const int b = blockIdx.x / kCluster;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  griddep_wait();

  const int64_t lo_b = a.cu_seqlens[b];
  const int64_t n_b = (int64_t)a.cu_seqlens[b + 1] - lo_b;
  const int64_t out_b = a.cu_kept[b];
  const int64_t k_b = (int64_t)a.cu_kept[b + 1] - out_b;

  const int64_t cchunk = (n_b + kCluster - 1) / kCluster;
  const int64_t c_lo = lo_b + (int64_t)crank * cchunk;
  int64_t c_hi = c_lo + cchunk;
  if (c_hi > lo_b + n_b) c_hi = lo_b + n_b;
  const int64_t c_len = c_hi > c_lo ? c_hi - c_lo : 0;
  int64_t wchunk = (c_len + kWarps - 1) / kWarps;
  wchunk = (wchunk + 31) & ~(int64_t)31;
  const int64_t w_lo = c_lo + (int64_t)warp * wchunk;
  int64_t w_hi = w_lo + wchunk;
  if (w_hi > c_hi) w_hi = c_hi;
  const bool cached = c_len <= kSmemKeys;

  // ---- pass 0: keys into shared memory, count non-prunable tokens
  uint32_t q_cnt = 0;
  for (int64_t base = w_lo; base < w_hi; base += 32) {
    const int64_t j = base + lane;
    const bool valid = j < w_hi;
    uint8_t p = 0;
    uint32_t key = 0;
    if (valid) {
      p = a.prunable[j];
      key = order_key(a.z[j]);
      if (cached) {
        S.keys[j - c_lo] = key;
        S.pr[j - c_lo] = p;
      }
    }
    q_cnt += __popc(__ballot_sync(0xFFFFFFFFu, valid && !p));
  }
  if (lane == 0) S.warp_cnt[warp][0] = q_cnt;
  __syncthreads();
  if (tid == 0) {
    uint32_t t = 0;
    for (int w = 0; w < kWarps; ++w) t += S.warp_cnt[w][0];
    S.xchg[0] = t;
  }
  cluster.sync();
  uint32_t q_b = 0;
  for (int r = 0; r < kCluster; ++r) q_b += cluster.map_shared_rank(&S.xchg[0], r)[0];
  const int64_t d_b = n_b - q_b;
  const int64_t kd = k_b - (int64_t)q_b;
  const bool bad = kd < 0 || kd > d_b;
  cluster.sync();  // every CTA has read xchg[0] before it is reused
  if (bad) {
    if (crank == 0 && tid == 0 && a.status) atomicOr(a.status, TG_STATUS_BUDGET);
    return;  // uniform across the cluster; no further shared-memory exchange
  }

  auto key_at = [&](int64_t j, uint32_t& key, uint8_t& p) {
    if (cached) {
      key = S.keys[j - c_lo];
      p = S.pr[j - c_lo];
    } else {
      key = order_key(a.z[j]);
      p = a.prunable[j];
    }
  };

  // ---- radix select of the kd-th largest prunable key
  uint32_t thr = 0xFFFFFFFFu;  // unreachable: no token ties or exceeds it when kd == 0
  uint32_t need = 0;
  if (kd > 0) {
    uint32_t prefix = 0, pmask = 0;
    need = (uint32_t)kd;
    const int shifts[3] = {21, 10, 0};
    const int nbins[3] = {2048, 2048, 1024};
    for (int pass = 0; pass < 3; ++pass) {
      const int sh = shifts[pass], nb = nbins[pass];
      uint32_t* hist = S.hist[pass & 1];
      for (int i = tid; i < kBins; i += kThreads) hist[i] = 0;
      __syncthreads();
      for (int64_t base = w_lo; base < w_hi; base += 32) {
        const int64_t j = base + lane;
        uint32_t key = 0;
        uint8_t p = 0;
        if (j < w_hi) key_at(j, key, p);
        const bool cand = (j < w_hi) && p && ((key & pmask) == prefix);
        const uint32_t bin = cand ? ((key >> sh) & (uint32_t)(nb - 1)) : 0xFFFFFFFFu;
        const uint32_t peers = __match_any_sync(0xFFFFFFFFu, bin);
        if (cand && (peers & lt_mask) == 0) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
      }
      cluster.sync();
      for (int i = tid; i < nb; i += kThreads) {
        uint32_t t = 0;
        for (int r = 0; r < kCluster; ++r) t += cluster.map_shared_rank(hist, r)[i];
        S.tot[i] = t;
      }
      __syncthreads();
      // thread t owns bins [4t, 4t+4) (nb <= 4 * kThreads)
      uint32_t mine = 0;
      for (int i = 0; i < 4; ++i) {
        const int bi = 4 * tid + i;
        if (bi < nb) mine += S.tot[bi];
      }
      uint32_t above = block_suffix_excl(mine, S.scan);
      for (int i = 3; i >= 0; --i) {
        const int bi = 4 * tid + i;
        if (bi >= nb) continue;
        const uint32_t c = S.tot[bi];
        if (above < need && above + c >= need) {
          S.sel_bin = (uint32_t)bi;
          S.count_above = above;
        }
        above += c;
      }
      __syncthreads();
      prefix |= S.sel_bin << sh;
      pmask |= (uint32_t)(nb - 1) << sh;
      need -= S.count_above;
      __syncthreads();
    }
    thr = prefix;
  }

  // ---- counting pass: per warp (q, gt, eq)
  uint32_t gt = 0, eq = 0, qq = 0;
  for (int64_t base = w_lo; base < w_hi; base += 32) {
    const int64_t j = base + lane;
    uint32_t key = 0;
    uint8_t p = 0;
    const bool valid = j < w_hi;
    if (valid) key_at(j, key, p);
    gt += __popc(__ballot_sync(0xFFFFFFFFu, valid && p && key > thr));
    eq += __popc(__ballot_sync(0xFFFFFFFFu, valid && p && key == thr));
    qq += __popc(__ballot_sync(0xFFFFFFFFu, valid && !p));
  }
  if (lane == 0) {
    S.warp_cnt[warp][0] = qq;
    S.warp_cnt[warp][1] = gt;
    S.warp_cnt[warp][2] = eq;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t t0 = 0, t1 = 0, t2 = 0;
    for (int w = 0; w < kWarps; ++w) {
      t0 += S.warp_cnt[w][0];
      t1 += S.warp_cnt[w][1];
      t2 += S.warp_cnt[w][2];
    }
    S.xchg[0] = t0;
    S.xchg[1] = t1;
    S.xchg[2] = t2;
  }
  cluster.sync();
  if (tid == 0) {
    // ties go to the lowest indices: CTAs in rank order, warps in index order
    uint32_t eq_before = 0, kept_before = 0;
    uint32_t my_sel_eq = 0;
    for (int r = 0; r < kCluster; ++r) {
      const uint32_t* x = cluster.map_shared_rank(S.xchg, r);
      const uint32_t rq = x[0], rgt = x[1], req = x[2];
      const uint32_t left = need > eq_before ? need - eq_before : 0u;
      const uint32_t sel = left < req ? left : req;
      if (r == crank) {
        my_sel_eq = sel;
        break;
      }
      kept_before += rq + rgt + sel;
      eq_before += req;
    }
    uint32_t weq_before = 0, out = (uint32_t)out_b + kept_before;
    for (int w = 0; w < kWarps; ++w) {
      const uint32_t left = my_sel_eq > weq_before ? my_sel_eq - weq_before : 0u;
      const uint32_t sel = left < S.warp_cnt[w][2] ? left : S.warp_cnt[w][2];
      S.warp_sel_eq[w] = sel;
      S.warp_out[w] = out;
      out += S.warp_cnt[w][0] + S.warp_cnt[w][1] + sel;
      weq_before += S.warp_cnt[w][2];
    }
  }
  cluster.sync();  // last distributed-shared-memory access is above

  // ---- write pass: ballot compaction in position order
  const uint32_t sel_eq = S.warp_sel_eq[warp];
  uint32_t out = S.warp_out[warp];
  uint32_t eq_seen = 0;
  for (int64_t base = w_lo; base < w_hi; base += 32) {
    const int64_t j = base + lane;
    uint32_t key = 0;
    uint8_t p = 0;
    const bool valid = j < w_hi;
    if (valid) key_at(j, key, p);
    const bool is_eq = valid && p && key == thr;
    const uint32_t eq_mask = __ballot_sync(0xFFFFFFFFu, is_eq);
    const uint32_t my_rank = eq_seen + __popc(eq_mask & lt_mask);
    const bool sel = valid && p && (key > thr || (is_eq && my_rank < sel_eq));
    const bool kept = valid && (!p || sel);
    const uint32_t kmask = __ballot_sync(0xFFFFFFFFu, kept);
    if (kept) {
      const uint32_t slot = out + __popc(kmask & lt_mask);
      a.kept_idx[slot] = (int32_t)j;
      a.kept_pos[slot] = (int32_t)(j - lo_b);
      a.kept_bias[slot] = p ? a.z[j] : 0.0f;
    }
    eq_seen += __popc(eq_mask);
    out += __popc(kmask);
  }
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" int tg_topk_compact(const float* z, const uint8_t* prunable, const int32_t* cu_seqlens,
                               const int32_t* cu_seqlens_host, const int32_t* cu_kept,
                               const int32_t* cu_kept_host, int batch, int32_t* kept_idx,
                               int32_t* kept_pos, float* kept_bias, uint32_t* status,
                               tg_stream_t stream) {
  if (batch < 0 || !cu_seqlens_host || !cu_kept_host) return TG_ERR_INVALID_ARGUMENT;
  if (batch == 0) return TG_OK;
  if (!cu_seqlens || !cu_kept) return TG_ERR_INVALID_ARGUMENT;
  if (cu_seqlens_host[0] != 0 || cu_kept_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    const int64_t k = (int64_t)cu_kept_host[b + 1] - cu_kept_host[b];
    if (n < 0 || k < 0 || k > n) return TG_ERR_INVALID_ARGUMENT;
  }
  const int64_t total = cu_seqlens_host[batch];
  const int64_t kept = cu_kept_host[batch];
  if (total > 0 && (!z || !prunable)) return TG_ERR_INVALID_ARGUMENT;
  if (kept > 0 && (!kept_idx || !kept_pos || !kept_bias)) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  const size_t smem = sizeof(Shared);
  static bool attr_done = false;
  if (!attr_done) {
    TG_CUDA_TRY(cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem));
    attr_done = true;
  }
  TopkArgs a{z, prunable, cu_seqlens, cu_kept, kept_idx, kept_pos, kept_bias, status};
  return launch(topk_kernel, dim3((unsigned)(batch * kCluster)), dim3(kThreads), smem,
                (cudaStream_t)stream, a);
}
