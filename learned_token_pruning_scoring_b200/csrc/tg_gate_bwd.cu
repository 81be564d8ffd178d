// Backward of the gate's scorer: its parameter gradients from dL/d(kept_bias).
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 门控到底插在模型的哪个位置 (a small MLP scores each token's normalised residual; the
// scores are RMSNorm-normalised along the sequence and become the attention bias) and
// section 端到端训练的关键在 token 门控注意力 (the gate learns end to end through the gated
// attention, whose backward gives the gradient of the bias).
//
// With r_t = 1 / rms(h_t), u_t = W1 (r_t h_t * norm_w), s_t = sum_f w2_f SiLU(u_tf) and
// z_t = s_t / rms_b over request b (the top-K choice is piecewise constant and passes
// no gradient):
//   dz_t  = d_kept_bias[r] where t = kept_idx[r] is prunable, else 0
//   ds_t  = (dz_t - z_t m_b) / rms_b,  m_b = (1 / N_b) sum over the request of dz z
//   dw2_f = sum_t ds_t SiLU(u_tf)
//   du_tf = ds_t w2_f SiLU'(u_tf)
//   M[i, f] = sum_t h_ti (r_t du_tf),  dW1[f, i] = norm_w_i M[i, f],
//   dnorm_w_i = sum_f W1[f, i] M[i, f]
// Kernels, in stream order:
//   1. prep: per request, rms_b from s and m_b from the kept rows (fixed order, the same
//      in every CTA of the request), then ds_t = -z_t m_b / rms_b on every row;
//   2. scatter: ds_t += dz_t / rms_b on the kept prunable rows (distinct rows);
//   3. the scorer GEMM again (tcgen05, the row RMS from the A stages as in the forward)
//      with a gradient epilogue: du'_t = r_t du_t as bf16 [T, 256] and per-32-row
//      column sums of ds_t SiLU(u_tf);
//   4. weight gradient M = h^T du' on tcgen05, both operands MN-major (the tokens, the
//      contraction index, are the rows of h and du'), one 128-feature tile of M per CTA
//      and the tokens split into S slices of whole 64-token steps; each CTA writes its
//      fp32 partial of M as [f][i];
//   5. finish: M from the S partials in slice order, dW1, and per-16-feature partial
//      sums of dnorm_w;
//   6. column sums of the dw2 chunk partials in fixed groups;
//   7. final: dnorm_w and dw2 from their partials in order.
// Every reduction runs in a fixed order, so the results are bit-reproducible.
#include <cstdint>

#include "tg_host.h"
#include "tg_ptx.cuh"

namespace tg {
namespace {

constexpr int kWidth = 256;
constexpr int kPrepThreads = 256;
constexpr int kPrepRowsPerCta = 8192;
constexpr int kScatterThreads = 256;

// recompute GEMM (u = W1' h_t per 128-row tile, all 256 scorer features)
constexpr int kGgBM = 128;
constexpr int kGgBK = 64;
constexpr int kGgStages = 4;
constexpr int kGgABytes = kGgBM * kGgBK * 2;             // 16 KB
constexpr int kGgBBytes = kWidth * kGgBK * 2;            // 32 KB
constexpr int kGgStageBytes = kGgABytes + kGgBBytes;
constexpr int kGgBarBytes = 256;
constexpr int kGgSmem = 1024 + kGgStages * kGgStageBytes + kGgBarBytes + kWidth * 4;
constexpr int kGgThreads = 192;

// weight-gradient GEMM tiles
constexpr int kWgBM = 128;                          // hidden features per CTA (MMA M)
constexpr int kWgBK = 64;                           // tokens per stage (MMA K, 4 steps of 16)
constexpr int kWgStages = 4;
constexpr int kWgBox = kWgBK * 128;                 // 64 token rows x 64 bf16 columns: 8 KB
constexpr int kWgABytes = 2 * kWgBox;               // h: 128 features
constexpr int kWgBBytes = (kWidth / 64) * kWgBox;   // du': 256 features
constexpr int kWgStageBytes = kWgABytes + kWgBBytes;
constexpr int kWgSmem = 1024 + kWgStages * kWgStageBytes + 256;
constexpr int kWgThreads = 192;
constexpr int kMaxSlices = 16;

constexpr int kFinFeatures = 16;                    // scorer features per finish block
constexpr int kDnParts = kWidth / kFinFeatures;
constexpr int kColGroups = 128;                     // groups of dw2 chunk partials

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__device__ double block_sum_in_order(double v, double* red) {
  // fixed shuffle tree inside each warp, then the warp totals in index order; every
  // thread returns the same total
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
  return t;
}

__global__ void __launch_bounds__(kPrepThreads)
    score_grad_prep_kernel(const float* __restrict__ s, const int32_t* __restrict__ cu,
                           const int32_t* __restrict__ ck, const int32_t* __restrict__ kept_idx,
                           const float* __restrict__ d_kept_bias,
                           const uint8_t* __restrict__ prunable, float eps,
                           float* __restrict__ ds, float* __restrict__ rms_out,
                           uint32_t* status) {
  __shared__ double red[kPrepThreads / 32];
  griddep_wait();
  const int b = blockIdx.y;
  const int64_t lo = cu[b], hi = cu[b + 1];
  const int64_t n = hi - lo;
  const int64_t my_lo = lo + (int64_t)blockIdx.x * kPrepRowsPerCta;
  if (n <= 0 || my_lo >= hi) return;
  const int tid = threadIdx.x;
  double acc = 0.0;
  for (int64_t j = lo + tid; j < hi; j += kPrepThreads) acc += (double)s[j] * s[j];
  const float rms = (float)sqrt(block_sum_in_order(acc, red) / (double)n + (double)eps);
  __syncthreads();  // every thread has read red before it is reused
  double dzz = 0.0;  // sum of dz z over the request: only kept prunable rows have dz != 0
  for (int64_t r = (int64_t)ck[b] + tid; r < ck[b + 1]; r += kPrepThreads) {
    const int64_t t = kept_idx[r];
    if (t < lo || t >= hi) {
      if (status && blockIdx.x == 0) atomicOr(status, TG_STATUS_BOUNDS);
      continue;
    }
    if (prunable[t]) dzz += (double)d_kept_bias[r] * (double)(s[t] / rms);
  }
  const float m = (float)(block_sum_in_order(dzz, red) / (double)n);
  if (blockIdx.x == 0 && tid == 0) rms_out[b] = rms;
  int64_t my_hi = my_lo + kPrepRowsPerCta;
  if (my_hi > hi) my_hi = hi;
  for (int64_t j = my_lo + tid; j < my_hi; j += kPrepThreads) ds[j] = -((s[j] / rms) * m) / rms;
}

__global__ void __launch_bounds__(kScatterThreads)
    score_grad_scatter_kernel(const int32_t* __restrict__ cu, const int32_t* __restrict__ ck,
                              const int32_t* __restrict__ kept_idx,
                              const float* __restrict__ d_kept_bias,
                              const uint8_t* __restrict__ prunable,
                              const float* __restrict__ rms, float* __restrict__ ds) {
  griddep_wait();
  const int b = blockIdx.y;
  const int64_t r = (int64_t)ck[b] + (int64_t)blockIdx.x * kScatterThreads + threadIdx.x;
  if (r >= ck[b + 1]) return;
  const int64_t t = kept_idx[r];
  if (t < cu[b] || t >= cu[b + 1]) return;  // reported by the prep kernel
  if (prunable[t]) ds[t] += d_kept_bias[r] / rms[b];
}

struct GradGemmParams {
  int64_t M;          // tokens
  int K;              // hidden
  float eps;          // of the row RMSNorm
  const float* w2;    // [256]
  const float* ds;    // [M]
  uint16_t* du;       // [M, 256] bf16: r_t ds_t w2_f SiLU'(u_tf)
  float* chunks;      // [ceil(M / 32), 256]: sum over each 32-row chunk of ds_t SiLU(u_tf)
  uint32_t* status;
};

// Sum over the warp's 32 lanes of each of 32 per-lane values, by recursive halving:
// at offset o every lane keeps half of its values and adds the partner's copy of that
// half, so after offsets 16, 8, 4, 2, 1 lane l holds the total of value l.  31 shuffles,
// and the order of the additions is fixed.
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  return v[0];
}

// The scorer GEMM of the forward (one CTA per 128 token rows, N = 256, K = hidden in
// 64-column k-blocks through a 4-stage TMA ring, 128-byte swizzle, K-major operands)
// with its gradient epilogue.  Roles: warp 0 lane 0 loads the h and W1' k-blocks;
// warp 1 owns TMEM and lane 0 issues the MMAs (M = 128, N = 256, K = 16); warps 2-5
// read every A stage for the row sums of squares (a stage is released by the MMA
// commit plus each of these 128 threads), then each thread takes one row of the accumulator:
// u = r acc, du' = r ds w2 SiLU'(u) stored as bf16, and the warp's column sums of
// ds SiLU(u) over its 32 rows.  Rows past M come from the TMA's zero fill with ds = 0.
__global__ void __launch_bounds__(kGgThreads, 1)
    score_grad_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB, GradGemmParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGgStages * kGgStageBytes);
  uint64_t* empty = full + kGgStages;
  uint64_t* acc_full = empty + kGgStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w2s = reinterpret_cast<float*>(smem + kGgStages * kGgStageBytes + kGgBarBytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * kGgBM;
  const int nk = p.K / kGgBK;

  if (tid == 0) {
    for (int s = 0; s < kGgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 128);  // the MMA commit and each of the 128 norm readers
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kWidth);
    tmem_relinquish();
  }
  griddep_wait();  // ds comes from the grid before this one
  for (int i = tid; i < kWidth; i += kGgThreads) w2s[i] = p.w2[i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kGgStages;
        const uint32_t ph = (uint32_t)(kb / kGgStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) break;
        unsigned char* a_s = tiles + s * kGgStageBytes;
        mbar_arrive_expect_tx(&full[s], kGgStageBytes);
        tma_load_2d(a_s, &tmA, kb * kGgBK, (int32_t)m0, &full[s]);
        tma_load_2d(a_s + kGgABytes, &tmB, kb * kGgBK, 0, &full[s]);
        ++issued;
      }
      // never leave the CTA with bulk copies still landing in its shared memory
      for (int kb = issued - kGgStages < 0 ? 0 : issued - kGgStages; kb < issued; ++kb)
        mbar_wait(&full[kb % kGgStages], (uint32_t)(kb / kGgStages) & 1u, nullptr, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kGgBM, kWidth, false, false);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kGgStages;
        const uint32_t ph = (uint32_t)(kb / kGgStages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + s * kGgStageBytes);
        const uint32_t b_addr = a_addr + kGgABytes;
#pragma unroll
        for (int k = 0; k < kGgBK / 16; ++k)
          mma_ss(tmem, sw128_desc(a_addr + k * 32, 16, 1024),
                 sw128_desc(b_addr + k * 32, 16, 1024), idesc, (kb | k) != 0);
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.status);  // all MMAs retired before TMEM is freed
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    const int64_t grow = m0 + row;
    const bool live = grow < p.M;
    float ss = 0.f;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % kGgStages;
      const uint32_t ph = (uint32_t)(kb / kGgStages) & 1u;
      if (!warp_all(mbar_wait(&full[s], ph, abort_flag, p.status))) break;
      const unsigned char* rowp = tiles + s * kGgStageBytes + row * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        // the row's eight 16-byte chunks, XOR-ordered so a quarter-warp hits distinct banks
        const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((j ^ (row & 7)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          ss = fmaf(f.x, f.x, ss);
          ss = fmaf(f.y, f.y, ss);
        }
      }
      // each reader releases the stage itself (its reads ordered before the refill)
      fence_proxy_async_smem();
      mbar_arrive(&empty[s]);
    }
    const float rscale = rsqrtf(ss / (float)p.K + p.eps);
    const bool ok = warp_all(mbar_wait(acc_full, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok) {
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
      const int64_t chunk_row = m0 + q * 32;  // first row of this warp's 32-row chunk
      const float dsr = live ? p.ds[grow] : 0.f;
      const float g = dsr * rscale;
#pragma unroll 1
      for (int c = 0; c < kWidth / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_wait_ld();
        float a[32];
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float d2[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const float u = __uint_as_float(r[i + e]) * rscale;
            const float sg = 1.0f / (1.0f + __expf(-u));
            a[i + e] = dsr * (u * sg);
            d2[e] = g * w2s[c * 32 + i + e] * (sg * (1.0f + u * (1.0f - sg)));
          }
          w[i >> 1] = pack_bf16x2(d2[0], d2[1]);
        }
        if (live) {
          uint4* dp = reinterpret_cast<uint4*>(p.du + grow * kWidth + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            dp[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
        const float col = warp_transpose_sum(a, lane);
        if (chunk_row < p.M) p.chunks[(chunk_row >> 5) * (int64_t)kWidth + c * 32 + lane] = col;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kWidth);
  }
}

// M partials: CTA (x, y) accumulates features i0 = 128 x .. i0 + 127 against all 256
// scorer features over the token steps of slice y, in TMEM (128 lanes = i, 256 columns
// = f).  Roles: warp 0 lane 0 streams the h and du' tiles (TMA, 128-byte swizzle; rows
// past the last token read as zero), warp 1 owns TMEM and lane 0 issues the MMAs,
// warps 2-5 write the accumulator to partial[y][f][i] (one TMEM lane quarter each).
// A stage holds h rows t0 .. t0 + 63 as two boxes of 64 features and du' rows t0 ..
// t0 + 63 as four boxes of 64 features; in both the features are the contiguous (MN)
// dimension: 64-wide atoms LBO = one box apart, 8-token groups SBO = 1024 bytes apart,
// and each 16-token MMA step starts 2048 bytes further into every box.
__global__ void __launch_bounds__(kWgThreads, 1)
    score_wgrad_kernel(const __grid_constant__ CUtensorMap tmH,
                       const __grid_constant__ CUtensorMap tmU, int steps_per_slice,
                       int total_steps, int hidden, float* __restrict__ partial,
                       uint32_t* status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWgStages * kWgStageBytes);
  uint64_t* empty = full + kWgStages;
  uint64_t* acc_full = empty + kWgStages;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i0 = blockIdx.x * kWgBM;
  const int slice = blockIdx.y;
  const int k_first = slice * steps_per_slice;
  const int k_end = k_first + steps_per_slice < total_steps ? k_first + steps_per_slice
                                                            : total_steps;
  const int nk = k_end - k_first;  // >= 1: the host sizes the grid so no slice is empty

  if (tid == 0) {
    for (int s = 0; s < kWgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmU);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kWidth);
    tmem_relinquish();
  }
  griddep_wait();  // du' comes from the grid before this one
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kWgStages;
        const uint32_t ph = (uint32_t)(kb / kWgStages) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, status)) break;
        unsigned char* st = tiles + s * kWgStageBytes;
        const int32_t t0 = (int32_t)((k_first + kb) * kWgBK);
        mbar_arrive_expect_tx(&full[s], kWgStageBytes);
        tma_load_2d(st, &tmH, i0, t0, &full[s]);
        tma_load_2d(st + kWgBox, &tmH, i0 + 64, t0, &full[s]);
#pragma unroll
        for (int j = 0; j < kWidth / 64; ++j)
          tma_load_2d(st + kWgABytes + j * kWgBox, &tmU, 64 * j, t0, &full[s]);
        ++issued;
      }
      // never leave the CTA with bulk copies still landing in its shared memory
      for (int kb = issued - kWgStages < 0 ? 0 : issued - kWgStages; kb < issued; ++kb)
        mbar_wait(&full[kb % kWgStages], (uint32_t)(kb / kWgStages) & 1u, nullptr, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kWgBM, kWidth, true, true);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % kWgStages;
        const uint32_t ph = (uint32_t)(kb / kWgStages) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + s * kWgStageBytes);
        const uint32_t b_addr = a_addr + kWgABytes;
#pragma unroll
        for (int k = 0; k < kWgBK / 16; ++k)
          mma_ss(tmem, sw128_desc(a_addr + k * 2048, kWgBox, 1024),
                 sw128_desc(b_addr + k * 2048, kWgBox, 1024), idesc, (kb | k) != 0);
        mma_commit(&empty[s]);
      }
      mma_commit(acc_full);
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, status);  // all MMAs retired before TMEM is freed
    }
  } else {
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int i = i0 + q * 32 + lane;
    const bool ok = warp_all(mbar_wait(acc_full, 0, abort_flag, status));
    tc_fence_after();
    if (ok) {
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
      float* out = partial + (int64_t)slice * kWidth * hidden + i;
#pragma unroll 1
      for (int c = 0; c < kWidth / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tbase + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) out[(int64_t)(c * 32 + j) * hidden] = __uint_as_float(r[j]);
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kWidth);
  }
}

__global__ void __launch_bounds__(128)
    score_wgrad_finish_kernel(const float* __restrict__ partial, int slices, int hidden,
                              const float* __restrict__ norm_w, const uint16_t* __restrict__ W1,
                              float* __restrict__ dW1, float* __restrict__ dn_part) {
  griddep_wait();
  const int i = blockIdx.x * 128 + threadIdx.x;  // hidden is a multiple of 128
  const int f0 = blockIdx.y * kFinFeatures;
  const float nw = norm_w ? norm_w[i] : 1.0f;
  float dn = 0.f;
  for (int f = f0; f < f0 + kFinFeatures; ++f) {
    float m = 0.f;
    for (int sl = 0; sl < slices; ++sl) m += partial[((int64_t)sl * kWidth + f) * hidden + i];
    dW1[(int64_t)f * hidden + i] = m * nw;
    dn = fmaf(__uint_as_float((uint32_t)W1[(int64_t)f * hidden + i] << 16), m, dn);
  }
  dn_part[(int64_t)blockIdx.y * hidden + i] = dn;
}

__global__ void __launch_bounds__(kWidth)
    column_sums_kernel(const float* __restrict__ chunks, int64_t n_chunks, int64_t per_group,
                       float* __restrict__ out) {
  griddep_wait();
  const int f = threadIdx.x;
  const int64_t c0 = (int64_t)blockIdx.x * per_group;
  const int64_t c1 = c0 + per_group < n_chunks ? c0 + per_group : n_chunks;
  float acc = 0.f;
  for (int64_t c = c0; c < c1; ++c) acc += chunks[c * kWidth + f];
  out[(int64_t)blockIdx.x * kWidth + f] = acc;
}

__global__ void __launch_bounds__(kWidth)
    score_grad_final_kernel(const float* __restrict__ dn_part, int hidden,
                            const float* __restrict__ dw2_part, int groups,
                            float* __restrict__ dnorm_w, float* __restrict__ dw2) {
  griddep_wait();
  const int tid = threadIdx.x;
  if (dnorm_w) {
    for (int i = tid; i < hidden; i += kWidth) {
      double a = 0.0;
      for (int g = 0; g < kDnParts; ++g) a += (double)dn_part[(int64_t)g * hidden + i];
      dnorm_w[i] = (float)a;
    }
  }
  double a = 0.0;
  for (int g = 0; g < groups; ++g) a += (double)dw2_part[(int64_t)g * kWidth + tid];
  dw2[tid] = (float)a;
}

// Token slices of the weight-gradient GEMM: enough CTAs for one wave over the SMs, no
// slice empty.
void plan_slices(int64_t total_tokens, int hidden, int sms, int& steps, int& per, int& slices) {
  steps = (int)((total_tokens + kWgBK - 1) / kWgBK);
  const int tiles = hidden / kWgBM;
  int want = sms / tiles;
  if (want < 1) want = 1;
  if (want > kMaxSlices) want = kMaxSlices;
  if (want > steps) want = steps;
  per = (steps + want - 1) / want;
  slices = (steps + per - 1) / per;
}

struct Layout {
  size_t w1f, du, chunks, partial, dn, dw2p, rms, total;
};

Layout layout(int64_t total_tokens, int hidden, int batch) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  const int64_t steps = (total_tokens + kWgBK - 1) / kWgBK;
  const int64_t max_slices = steps < kMaxSlices ? steps : kMaxSlices;
  L.w1f = take((size_t)kWidth * hidden * 2);
  L.du = take((size_t)total_tokens * kWidth * 2);
  L.chunks = take((size_t)((total_tokens + 31) / 32) * kWidth * 4);
  L.partial = take((size_t)max_slices * kWidth * hidden * 4);
  L.dn = take((size_t)kDnParts * hidden * 4);
  L.dw2p = take((size_t)kColGroups * kWidth * 4);
  L.rms = take((size_t)(batch > 0 ? batch : 1) * 4);
  L.total = off;
  return L;
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" size_t tg_gate_score_backward_workspace_size(int64_t total_tokens, int hidden,
                                                        int width, int batch) {
  if (total_tokens < 0 || hidden <= 0 || width != kWidth || batch < 0) return 0;
  return layout(total_tokens, hidden, batch).total;
}

extern "C" int tg_gate_score_backward(
    const tg_bf16* h, int64_t ld_h, int64_t total_tokens, int hidden, const float* norm_w,
    const tg_bf16* W1, int width, const float* w2, float eps_norm, const float* s,
    const int32_t* cu_seqlens, const int32_t* cu_seqlens_host, int batch, float eps_seq,
    const uint8_t* prunable, const int32_t* cu_kept, const int32_t* cu_kept_host,
    const int32_t* kept_idx, const float* d_kept_bias, float* ds_out, float* dW1,
    float* dnorm_w, float* dw2, void* workspace, size_t workspace_bytes, uint32_t* status,
    tg_stream_t stream) {
  if (width != kWidth || hidden <= 0 || (hidden % kWgBM)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (total_tokens < 0 || batch < 0 || !cu_seqlens_host || !cu_kept_host)
    return TG_ERR_INVALID_ARGUMENT;
  if (!(eps_norm >= 0.f) || !(eps_seq >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (batch == 0 && total_tokens != 0) return TG_ERR_INVALID_ARGUMENT;
  if (batch > 0) {
    if (cu_seqlens_host[0] != 0 || cu_seqlens_host[batch] != total_tokens || cu_kept_host[0] != 0)
      return TG_ERR_INVALID_ARGUMENT;
  }
  int64_t max_n = 0, max_k = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_seqlens_host[b + 1] - cu_seqlens_host[b];
    const int64_t k = (int64_t)cu_kept_host[b + 1] - cu_kept_host[b];
    if (n < 0 || k < 0 || k > n) return TG_ERR_INVALID_ARGUMENT;
    if (n > max_n) max_n = n;
    if (k > max_k) max_k = k;
  }
  if (!dW1 || !dw2) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  cudaStream_t st = (cudaStream_t)stream;
  if (total_tokens == 0) {  // no tokens: every gradient is zero
    TG_CUDA_TRY(cudaMemsetAsync(dW1, 0, (size_t)kWidth * hidden * 4, st));
    TG_CUDA_TRY(cudaMemsetAsync(dw2, 0, (size_t)kWidth * 4, st));
    if (dnorm_w) TG_CUDA_TRY(cudaMemsetAsync(dnorm_w, 0, (size_t)hidden * 4, st));
    return TG_OK;
  }
  if (!h || !W1 || !w2 || !s || !cu_seqlens || !prunable || !cu_kept || !ds_out ||
      (cu_kept_host[batch] > 0 && (!kept_idx || !d_kept_bias)))
    return TG_ERR_INVALID_ARGUMENT;
  if (ld_h < hidden) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(h) || !aligned16(W1) || !stride_ok(ld_h, 2)) return TG_ERR_MISALIGNED;
  const Layout L = layout(total_tokens, hidden, batch);
  if (!workspace || workspace_bytes < L.total || !aligned16(workspace)) return TG_ERR_WORKSPACE;

  unsigned char* ws = static_cast<unsigned char*>(workspace);
  uint16_t* w1f = reinterpret_cast<uint16_t*>(ws + L.w1f);
  uint16_t* du = reinterpret_cast<uint16_t*>(ws + L.du);
  float* chunks = reinterpret_cast<float*>(ws + L.chunks);
  float* partial = reinterpret_cast<float*>(ws + L.partial);
  float* dn_part = reinterpret_cast<float*>(ws + L.dn);
  float* dw2_part = reinterpret_cast<float*>(ws + L.dw2p);
  float* rms = reinterpret_cast<float*>(ws + L.rms);

  // 1-2: ds
  TG_TRY(launch(score_grad_prep_kernel,
                dim3((unsigned)((max_n + kPrepRowsPerCta - 1) / kPrepRowsPerCta), (unsigned)batch),
                dim3(kPrepThreads), 0, st, s, cu_seqlens, cu_kept, kept_idx, d_kept_bias,
                prunable, eps_seq, ds_out, rms, status));
  if (max_k > 0)
    TG_TRY(launch(score_grad_scatter_kernel,
                  dim3((unsigned)((max_k + kScatterThreads - 1) / kScatterThreads),
                       (unsigned)batch),
                  dim3(kScatterThreads), 0, st, cu_seqlens, cu_kept, kept_idx, d_kept_bias,
                  prunable, (const float*)rms, ds_out));

  // 3: u again, du' and the dw2 chunk sums
  const void* wmat = W1;
  if (norm_w) {
    TG_TRY(tg_fold_norm_weight(W1, hidden, kWidth, hidden, norm_w,
                               reinterpret_cast<tg_bf16*>(w1f), hidden, stream));
    wmat = w1f;
  }
  CUtensorMap ta, tb;
  TG_TRY(make_tmap_bf16_2d(&ta, h, (uint64_t)total_tokens, (uint64_t)hidden, (uint64_t)ld_h, 64,
                           128));
  TG_TRY(make_tmap_bf16_2d(&tb, wmat, (uint64_t)kWidth, (uint64_t)hidden, (uint64_t)hidden, 64,
                           256));
  GradGemmParams gp{};
  gp.M = total_tokens;
  gp.K = hidden;
  gp.eps = eps_norm;
  gp.w2 = w2;
  gp.ds = ds_out;
  gp.du = du;
  gp.chunks = chunks;
  gp.status = status;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  static int attr_dev = -1;
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(score_grad_gemm_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGgSmem));
    TG_CUDA_TRY(cudaFuncSetAttribute(score_wgrad_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kWgSmem));
    attr_dev = dev;
  }
  TG_TRY(launch(score_grad_gemm_kernel, dim3((unsigned)((total_tokens + kGgBM - 1) / kGgBM)),
                dim3(kGgThreads), kGgSmem, st, ta, tb, gp));

  // 4: M = h^T du' in token slices
  int steps = 0, per = 0, slices = 0;
  plan_slices(total_tokens, hidden, sm_count(), steps, per, slices);
  CUtensorMap th, tu;
  TG_TRY(make_tmap_bf16_2d(&th, h, (uint64_t)total_tokens, (uint64_t)hidden, (uint64_t)ld_h, 64,
                           kWgBK));
  TG_TRY(make_tmap_bf16_2d(&tu, du, (uint64_t)total_tokens, (uint64_t)kWidth, (uint64_t)kWidth,
                           64, kWgBK));
  TG_TRY(launch(score_wgrad_kernel, dim3((unsigned)(hidden / kWgBM), (unsigned)slices),
                dim3(kWgThreads), kWgSmem, st, th, tu, per, steps, hidden, partial, status));

  // 5-7: finish
  TG_TRY(launch(score_wgrad_finish_kernel, dim3((unsigned)(hidden / 128), (unsigned)kDnParts),
                dim3(128), 0, st, (const float*)partial, slices, hidden, norm_w,
                reinterpret_cast<const uint16_t*>(W1), dW1, dn_part));
  const int64_t n_chunks = (total_tokens + 31) / 32;
  const int64_t per_group = (n_chunks + kColGroups - 1) / kColGroups;
  const int groups = (int)((n_chunks + per_group - 1) / per_group);
  TG_TRY(launch(column_sums_kernel, dim3((unsigned)groups), dim3(kWidth), 0, st,
                (const float*)chunks, n_chunks, per_group, dw2_part));
  return launch(score_grad_final_kernel, dim3(1), dim3(kWidth), 0, st, (const float*)dn_part,
                hidden, (const float*)dw2_part, groups, dnorm_w, dw2);
}
