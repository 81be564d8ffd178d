// Gate scoring: fused RMSNorm + scoring MLP on tcgen05, then the sequence RMSNorm.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 门控到底插在模型的哪个位置 (a small MLP scores each token's normalised residual; the
// scores are RMSNorm-normalised along the sequence); "斯坦福与 UC Berkeley 提出 TokenGate：
// token 门控注意力让长上下文预填充最高快 11.3 倍", section "How does TokenGate learned token
// pruning work?" (the residual is the post-attention residual at the gate layer).
//
// Kernel 1: h[T, H] x W1[F, H]^T with F = 256 on the tensor cores; the epilogue applies
//   the row RMS, SiLU and the dot with w2, writes s[T] and the sum of s^2 over each
//   32-row chunk.  Two kernels compute it: the CTA-pair scorer below (the default) and
//   the one-CTA GEMM with its score epilogue (tg_gemm.cuh), selected by
//   tg_set_scorer_pair; both give the same s bit for bit (same products, same order).
// Kernel 2: per request, the chunk sums inside the request plus the ragged edge rows
//   are reduced in a fixed order (every CTA of the request computes the identical
//   total), then z = s / rms and bias = z on prunable tokens.
#include <cstdint>

#include "tg_gemm.cuh"
#include "tg_host.h"

namespace tg {

template <int BN, int STAGES, int EPI>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                cudaStream_t stream);

namespace {

constexpr int kWidth = 256;
constexpr int kNormThreads = 256;
// Rows written per CTA.  Every CTA of a request recomputes the request's sum of squares
// (in a fixed order, so all agree bit for bit): from the 32-row chunk sums that is cheap
// and small CTAs spread the work; without chunk sums each CTA rereads the whole request,
// so there the CTAs stay large.
constexpr int kNormRowsPerCta = 512;
constexpr int kNormRowsPerCtaNoPartials = 8192;

__global__ void fold_norm_kernel(const uint16_t* __restrict__ W1, const float* __restrict__ w,
                                 uint16_t* __restrict__ out, int width, int hidden) {
  griddep_wait();
  const int64_t n = (int64_t)width * hidden;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const float v = __uint_as_float((uint32_t)W1[i] << 16) * w[i % hidden];
    __nv_bfloat16 b = __float2bfloat16_rn(v);
    out[i] = *reinterpret_cast<uint16_t*>(&b);
  }
}

__device__ double block_sum_fixed(double v, double* red) {
  // fixed shuffle tree inside each warp, then warp totals in index order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(kNormThreads)
    seq_norm_kernel(const float* __restrict__ s, const float* __restrict__ partial,
                    const int32_t* __restrict__ cu, const uint8_t* __restrict__ prunable,
                    float eps, float* __restrict__ z, float* __restrict__ bias,
                    int rows_per_cta) {
  __shared__ double red[kNormThreads / 32];
  griddep_wait();
  const int b = blockIdx.y;
  const int64_t lo = cu[b], hi = cu[b + 1];
  const int64_t n = hi - lo;
  const int64_t my_lo = lo + (int64_t)blockIdx.x * rows_per_cta;
  if (n <= 0 || my_lo >= hi) return;
  const int tid = threadIdx.x;
  const int64_t c_first = (lo + 31) >> 5, c_last = hi >> 5;  // whole chunks [c_first, c_last)
  double acc = 0.0;
  if (partial && c_first < c_last) {
    for (int64_t c = c_first + tid; c < c_last; c += kNormThreads) acc += (double)partial[c];
    for (int64_t j = lo + tid; j < (c_first << 5); j += kNormThreads) acc += (double)s[j] * s[j];
    for (int64_t j = (c_last << 5) + tid; j < hi; j += kNormThreads) acc += (double)s[j] * s[j];
  } else {
    for (int64_t j = lo + tid; j < hi; j += kNormThreads) acc += (double)s[j] * s[j];
  }
  const double total = block_sum_fixed(acc, red);
  const float rms = (float)sqrt(total / (double)n + (double)eps);
  int64_t my_hi = my_lo + rows_per_cta;
  if (my_hi > hi) my_hi = hi;
  for (int64_t j = my_lo + tid; j < my_hi; j += kNormThreads) {
    const float zz = s[j] / rms;
    z[j] = zz;
    bias[j] = prunable[j] ? zz : 0.0f;
  }
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------- CTA-pair scorer
//
// s_t = sum_f w2_f SiLU(r_t (W1' h_t)_f) on CTA pairs: a cluster of two CTAs owns 256
// token rows at a time (128 per CTA) and the whole scorer width N = 256; the even CTA
// issues tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16) that reads both CTAs' shared
// memory, so each CTA streams 16 KB of h and only 16 KB of W1' (its half of the 256
// scorer rows) per 64-column k-block, half the W1' traffic of a one-CTA tile.  Clusters
// are persistent over the row tiles with two TMEM accumulators, so a tile's epilogue runs
// under the next tile's mainloop.  Roles per CTA (320 threads):
//   warp 0     one thread streams the h and W1' k-blocks through a 6-stage ring; both
//              CTAs' bytes complete on the even CTA's stage barrier (no multicast);
//   warp 1     TMEM owner; in the even CTA one thread issues the MMAs, commits each
//              stage's consumption to both CTAs' `consumed` barriers and each tile's
//              accumulator to both CTAs' `acc_full`;
//   warps 2-5  row-norm readers: after a stage is consumed each reads its row's 64 values
//              (sum of squares) and releases the stage itself (proxy fence + its own
//              arrive), then hands the tile's row sum of squares to the epilogue;
//   warps 6-9  epilogue, one TMEM lane quarter each (thread = row): r = rsqrt(mean h^2 +
//              eps), the SiLU reduction with w2, s and per-32-row sums of s^2.
constexpr int kSpStages = 6;
constexpr int kSpBK = 64;
constexpr int kSpABytes = 128 * kSpBK * 2;  // 128 rows of h
constexpr int kSpBBytes = 128 * kSpBK * 2;  // 128 of the 256 rows of W1'
constexpr int kSpStageBytes = kSpABytes + kSpBBytes;
constexpr int kSpThreads = 320;
constexpr int kSpRing = kSpStages * kSpStageBytes;
constexpr int kSpW2 = kSpRing;              // 256 floats
constexpr int kSpSS = kSpW2 + 1024;         // [2][128] row sums of squares
constexpr int kSpBar = kSpSS + 1024;
constexpr int kSpSmem = kSpBar + 256 + 1024;  // + alignment slack

struct ScorerArgs {
  int64_t M;
  int K;
  float eps;
  const float* w2;
  float* s_out;
  float* partial;  // [ceil(M / 32)]: sum of s^2 over each 32-row chunk
  uint32_t* status;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kSpThreads, 1)
    scorer_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, ScorerArgs p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = smem;
  float* w2s = reinterpret_cast<float*>(smem + kSpW2);
  float* ssb = reinterpret_cast<float*>(smem + kSpSS);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSpBar);
  uint64_t* consumed = full + kSpStages;
  uint64_t* empty = consumed + kSpStages;
  uint64_t* acc_full = empty + kSpStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2] (even CTA: one arrive per CTA)
  uint64_t* ss_full = acc_empty + 2;       // [2]
  uint64_t* ss_empty = ss_full + 2;        // [2]
  uint64_t* drain = ss_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = (int)(blockIdx.x >> 1), n_clusters = (int)(gridDim.x >> 1);
  const int n_tiles = (int)((p.M + 255) / 256);
  const int nk = p.K / kSpBK;

  if (tid == 0) {
    for (int s = 0; s < kSpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&consumed[s], 1);
      mbar_init(&empty[s], 128);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 2);
      mbar_init(&ss_full[b], 128);
      mbar_init(&ss_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  griddep_wait();  // h and the folded W1' may come from earlier grids
  for (int i = tid; i < kWidth; i += kSpThreads) w2s[i] = p.w2[i];
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full_lead0 = mapa_shared(smem_u32(&full[0]), 0);
      int kg = 0;
      bool ok = true;
      for (int t = cluster; ok && t < n_tiles; t += n_clusters) {
        const int32_t m0 = (int32_t)((int64_t)t * 256 + rank * 128);
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % kSpStages;
          const uint32_t ph = (uint32_t)(kg / kSpStages) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) {
            ok = false;
            break;
          }
          unsigned char* st = ring + s * kSpStageBytes;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kSpStageBytes);
          tma_load_2d_pair(st, &tmA, kb * kSpBK, m0, full_lead0 + s * 8);
          tma_load_2d_pair(st + kSpABytes, &tmB, kb * kSpBK, (int32_t)rank * 128,
                           full_lead0 + s * 8);
        }
      }
      // the even CTA waits until the last stages' bytes (both CTAs') have landed; the
      // odd CTA is held by the closing cluster barrier until then
      if (rank == 0)
        for (int g = kg - kSpStages < 0 ? 0 : kg - kSpStages; g < kg; ++g)
          mbar_wait(&full[g % kSpStages], (uint32_t)(g / kSpStages) & 1u, nullptr, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(256, kWidth, false, false);
      const uint32_t consumed_peer0 = mapa_shared(smem_u32(&consumed[0]), 1);
      const uint32_t acc_full_peer0 = mapa_shared(smem_u32(&acc_full[0]), 1);
      int kg = 0, i = 0;
      bool ok = true;
      for (int t = cluster; ok && t < n_tiles; t += n_clusters, ++i) {
        const int b = i & 1;
        if (!mbar_wait(&acc_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, p.status))
          break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(b * kWidth);
        for (int kb = 0; kb < nk; ++kb, ++kg) {
          const int s = kg % kSpStages;
          const uint32_t ph = (uint32_t)(kg / kSpStages) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, p.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(ring + s * kSpStageBytes);
          const uint32_t b_addr = a_addr + kSpABytes;
#pragma unroll
          for (int k = 0; k < kSpBK / 16; ++k)
            mma_ss_pair(d, sw128_desc(a_addr + k * 32, 16, 1024),
                        sw128_desc(b_addr + k * 32, 16, 1024), idesc, (kb | k) != 0);
          mma_commit_pair(smem_u32(&consumed[s]));
          mma_commit_pair(consumed_peer0 + s * 8);
        }
        if (!ok) break;
        mma_commit_pair(smem_u32(&acc_full[b]));
        mma_commit_pair(acc_full_peer0 + b * 8);
      }
      mma_commit_pair(smem_u32(drain));
      mbar_wait(drain, 0, nullptr, p.status);  // all MMAs (and their arrives) done
    }
  } else if (warp < 6) {
    // ---- row-norm readers: row (warp - 2) * 32 + lane of each tile
    const int row = (warp - 2) * 32 + lane;
    int kg = 0, i = 0;
    for (int t = cluster; t < n_tiles; t += n_clusters, ++i) {
      const int b = i & 1;
      float ss = 0.f;
      bool ok = true;
      for (int kb = 0; kb < nk; ++kb, ++kg) {
        const int s = kg % kSpStages;
        const uint32_t ph = (uint32_t)(kg / kSpStages) & 1u;
        if (!(ok = warp_all(mbar_wait(&consumed[s], ph, abort_flag, p.status)))) break;
        const unsigned char* rowp = ring + s * kSpStageBytes + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // the row's 16-byte chunks in XOR order: each quarter-warp on distinct banks
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((j ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
          }
        }
        fence_proxy_async_smem();  // these reads before the TMA write that refills the stage
        mbar_arrive(&empty[s]);
      }
      if (!ok) break;
      if (!warp_all(mbar_wait(&ss_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag,
                              p.status)))
        break;
      ssb[b * 128 + row] = ss;
      mbar_arrive(&ss_full[b]);
    }
  } else {
    // ---- epilogue: TMEM lane quarter warp & 3, thread = row
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t acc_empty_lead0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    int i = 0;
    for (int t = cluster; t < n_tiles; t += n_clusters, ++i) {
      const int b = i & 1;
      const uint32_t ph = (uint32_t)(i >> 1) & 1u;
      const int64_t m0 = (int64_t)t * 256 + rank * 128;
      const int64_t grow = m0 + row;
      bool ok = mbar_wait(&acc_full[b], ph, abort_flag, p.status) &&
                mbar_wait(&ss_full[b], ph, abort_flag, p.status);
      if (!named_bar_and(1, 128, ok)) break;
      tc_fence_after();
      const float rscale = rsqrtf(ssb[b * 128 + row] / (float)p.K + p.eps);
      mbar_arrive(&ss_empty[b]);
      const uint32_t tacc = tmem + (uint32_t)(b * kWidth) + ((uint32_t)(q * 32) << 16);
      float score = 0.f;
#pragma unroll 1
      for (int c = 0; c < kWidth / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tacc + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float u = __uint_as_float(r[e]) * rscale;
          score = fmaf(w2s[c * 32 + e], u / (1.0f + __expf(-u)), score);
        }
      }
      tc_fence_before();
      named_bar_sync(1, 128);  // all four warps are done with accumulator b
      if (warp == 6 && lane == 0) {
        if (rank == 0) mbar_arrive(&acc_empty[b]);
        else mbar_arrive_cluster(acc_empty_lead0 + b * 8);
      }
      if (grow < p.M) p.s_out[grow] = score;
      float sq = grow < p.M ? score * score : 0.f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
      if (lane == 0 && m0 + q * 32 < p.M) p.partial[(m0 + q * 32) >> 5] = sq;
    }
  }
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while the pair's MMAs or arrives may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

int launch_scorer_pair(const CUtensorMap& ta, const CUtensorMap& tb, const ScorerArgs& a,
                       cudaStream_t stream) {
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(scorer_pair_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSpSmem));
    attr_dev = dev;
  }
  const int64_t tiles = (a.M + 255) / 256;
  int clusters = sm_count() / 2;
  if (tiles < clusters) clusters = (int)tiles;
  return launch(scorer_pair_kernel, dim3((unsigned)(2 * clusters)), dim3(kSpThreads), kSpSmem,
                stream, ta, tb, a);
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" size_t tg_gate_score_workspace_size(int64_t total_tokens, int hidden, int width,
                                               int batch) {
  (void)batch;
  if (total_tokens < 0 || hidden <= 0 || width <= 0) return 0;
  const size_t fold = align256((size_t)width * hidden * 2);
  const size_t part = align256((size_t)((total_tokens + 31) / 32 + 1) * sizeof(float));
  return fold + part;
}

extern "C" int tg_gate_score(const tg_bf16* h, int64_t ld_h, int64_t total_tokens, int hidden,
                             const float* norm_w, const tg_bf16* W1, int width, const float* w2,
                             float eps_norm, const int32_t* cu_seqlens,
                             const int32_t* cu_seqlens_host, int batch, float eps_seq,
                             const uint8_t* prunable, float* s_out, float* z_out,
                             float* bias_out, void* workspace, size_t workspace_bytes,
                             uint32_t* status, tg_stream_t stream) {
  if (width != kWidth || hidden <= 0 || (hidden % 64)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (total_tokens < 0 || batch < 0 || !cu_seqlens_host) return TG_ERR_INVALID_ARGUMENT;
  if (!(eps_norm >= 0.f) || !(eps_seq >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (batch == 0) return total_tokens == 0 ? TG_OK : TG_ERR_INVALID_ARGUMENT;
  if (cu_seqlens_host[0] != 0 || cu_seqlens_host[batch] != total_tokens)
    return TG_ERR_INVALID_ARGUMENT;
  int64_t max_n = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    if (n < 0) return TG_ERR_INVALID_ARGUMENT;
    if (n > max_n) max_n = n;
  }
  if (total_tokens == 0) return TG_OK;
  if (!h || !W1 || !w2 || !cu_seqlens || !prunable || !s_out || !z_out || !bias_out)
    return TG_ERR_INVALID_ARGUMENT;
  if (ld_h < hidden) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(h) || !aligned16(W1) || !stride_ok(ld_h, 2)) return TG_ERR_MISALIGNED;
  const size_t need = tg_gate_score_workspace_size(total_tokens, hidden, width, batch);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return TG_ERR_WORKSPACE;
  TG_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  uint16_t* w1f = reinterpret_cast<uint16_t*>(ws);
  float* partial = reinterpret_cast<float*>(ws + align256((size_t)width * hidden * 2));

  const void* wmat = W1;
  if (norm_w) {
    const int64_t n = (int64_t)width * hidden;
    int grid = (int)((n + 255) / 256);
    if (grid > sm_count() * 8) grid = sm_count() * 8;
    TG_TRY(launch(fold_norm_kernel, dim3(grid), dim3(256), 0, st,
                  reinterpret_cast<const uint16_t*>(W1), norm_w, w1f, width, hidden));
    wmat = w1f;
  }
  CUtensorMap ta, tb;
  TG_TRY(make_tmap_bf16_2d(&ta, h, (uint64_t)total_tokens, (uint64_t)hidden, (uint64_t)ld_h, 64,
                           128));
  if (scorer_use_pair()) {
    TG_TRY(make_tmap_bf16_2d(&tb, wmat, (uint64_t)width, (uint64_t)hidden, (uint64_t)hidden, 64,
                             128));
    ScorerArgs sa{total_tokens, hidden, eps_norm, w2, s_out, partial, status};
    TG_TRY(launch_scorer_pair(ta, tb, sa, st));
    dim3 grid((unsigned)((max_n + kNormRowsPerCta - 1) / kNormRowsPerCta), (unsigned)batch);
    return launch(seq_norm_kernel, grid, dim3(kNormThreads), 0, st, (const float*)s_out,
                  (const float*)partial, cu_seqlens, prunable, eps_seq, z_out, bias_out,
                  kNormRowsPerCta);
  }
  TG_TRY(make_tmap_bf16_2d(&tb, wmat, (uint64_t)width, (uint64_t)hidden, (uint64_t)hidden, 64,
                           256));
  GemmParams p{};
  p.M = total_tokens;
  p.N = width;
  p.K = hidden;
  p.rmsnorm = 1;
  p.eps = eps_norm;
  p.w2 = w2;
  p.s_out = s_out;
  p.partial = partial;
  p.status = status;
  TG_TRY((launch_gemm<256, 4, EpiScore>(ta, tb, p, st)));

  dim3 grid((unsigned)((max_n + kNormRowsPerCta - 1) / kNormRowsPerCta), (unsigned)batch);
  return launch(seq_norm_kernel, grid, dim3(kNormThreads), 0, st, (const float*)s_out,
                (const float*)partial, cu_seqlens, prunable, eps_seq, z_out, bias_out,
                kNormRowsPerCta);
}

extern "C" int tg_seq_rmsnorm(const float* s, const int32_t* cu_seqlens,
                              const int32_t* cu_seqlens_host, int batch, const uint8_t* prunable,
                              float eps_seq, float* z_out, float* bias_out, tg_stream_t stream) {
  if (batch < 0 || !cu_seqlens_host || !(eps_seq >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (batch == 0) return TG_OK;
  if (cu_seqlens_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  int64_t max_n = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    if (n < 0) return TG_ERR_INVALID_ARGUMENT;
    if (n > max_n) max_n = n;
  }
  if (cu_seqlens_host[batch] == 0) return TG_OK;
  if (!s || !cu_seqlens || !prunable || !z_out || !bias_out) return TG_ERR_INVALID_ARGUMENT;
  if (z_out == s || bias_out == s) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  dim3 grid((unsigned)((max_n + kNormRowsPerCtaNoPartials - 1) / kNormRowsPerCtaNoPartials),
            (unsigned)batch);
  TG_TRY(launch(seq_norm_kernel, grid, dim3(kNormThreads), 0, (cudaStream_t)stream, s,
                (const float*)nullptr, cu_seqlens, prunable, eps_seq, z_out, bias_out,
                kNormRowsPerCtaNoPartials));
  return TG_OK;
}
