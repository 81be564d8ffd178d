// tcgen05 GEMMs C[M, N] = A[M, K] * W[N, K]^T for bf16 inputs with fp32 accumulation
// in tensor memory, fed by TMA through a shared-memory ring.
//
// gemm_kernel (one CTA per 128 x BN tile), 192 threads:
//   warp 0     one thread issues the TMA loads of A and W tiles (128-byte swizzle);
//   warp 1     allocates TMEM; one thread issues tcgen05.mma (M=128, N=BN, K=16);
//   warps 2-5  epilogue, one TMEM lane quarter each (thread = output row).  With a
//              folded RMSNorm they also read every A stage from shared memory during
//              the mainloop to accumulate the row's sum of squares, so the norm costs
//              no extra HBM pass: RMSNorm(a) W^T = r * (a W^T), r = 1/sqrt(mean a^2 + eps).
// gemm_pair_kernel (a cluster of two CTAs per 256 x 256 tile), same roles: each CTA
//   loads its 128 rows of A and its 128 rows of W; the even CTA issues the M=256 MMA
//   (tcgen05 cta_group::2) that reads both CTAs' shared memory and writes each CTA's
//   128 output rows into its own TMEM.  Per SM this halves the W bytes streamed per
//   MMA, so a 6-stage ring covers the load latency.  Both CTAs' loads (cta_group::2
//   TMA, no multicast) count their bytes on the even CTA's stage barrier, so the MMA
//   issuer sees one barrier per stage with no forwarding hop; the even CTA's commits
//   arrive on both CTAs' stage-free barriers.  A folded RMSNorm here
//   takes per-row sums of squares computed by the producer of A (row_ssq_in).
// Epilogues (per thread-row): EpiStore writes bf16 (+ residual, and optionally the
// sums of squares of the stored bf16 values per 128 columns); EpiScore reduces the row
// to s = sum_f w2[f] SiLU(r * acc[f]) and per-32-row partial sums of s^2; EpiQKV
// applies rotate-half RoPE at the row's position to the Q and K heads (pairs of
// columns 64 apart, from TMEM chunks c and c + 2) and routes Q, K and V tiles to their
// destinations (Q rows and the K and V rows of a compacted cache).
#pragma once
#include <cuda.h>

#include <cstdint>

#include "tg_ptx.cuh"

namespace tg {

enum { EpiStore = 0, EpiScore = 1, EpiQKV = 2, EpiSwiGLU = 3, EpiQKVNorm = 4 };

struct GemmParams {
  int64_t M;
  int N, K;
  int rmsnorm;
  float eps;
  // optional per-row sums of squares of A (K / 128 groups per row), used for the norm
  const float* row_ssq_in;
  int64_t ld_ssq_in;
  // EpiStore
  uint16_t* c;
  int64_t ldc;
  const uint16_t* residual;
  int64_t ldr;
  float* row_ssq_out;  // optional: sums of squares of the stored row, per 128 columns
  int64_t ld_ssq_out;
  // EpiScore
  const float* w2;
  float* s_out;
  float* partial;  // [ceil(M / 32)]
  // EpiQKV
  const int32_t* pos;     // [M] rotary position of each row, or null (see rope_row)
  const float* cos_sin;   // [max_pos, head_dim / 2, 2], or the per-row table if pos is null
  int max_pos;            // table rows, or the per-row table's row stride
  int q_cols, k_cols;     // Q heads in [0, q_cols), K heads in [q_cols, q_cols + k_cols)
  uint16_t* k_out;        // K rows: k_out + row * ld_kv (columns relative to q_cols)
  uint16_t* v_out;        // V rows: v_out + row * ld_kv (columns relative to q_cols + k_cols)
  int64_t ld_kv;
  // EpiQKVNorm (EpiQKV plus QK-norm, CTA-pair kernel only): per-head RMSNorm of the Q
  // and K heads before RoPE, weights [128] shared by the heads
  const float* q_norm_w;
  const float* k_norm_w;
  float qk_eps;
  uint32_t* status;
};

template <int BN, int STAGES>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int W2_BYTES = BN * 4;
  static constexpr int SMEM = 1024 + TILE_BYTES + BAR_BYTES + W2_BYTES;
  static constexpr int THREADS = 192;
};

// Row scale of the folded RMSNorm from per-row partial sums of squares.
__device__ __forceinline__ float rscale_from_ssq(const GemmParams& p, int64_t grow) {
  const float* ss = p.row_ssq_in + grow * p.ld_ssq_in;
  float t = 0.f;
  for (int g = 0; g < p.K / 128; ++g) t += ss[g];
  return rsqrtf(t / (float)p.K + p.eps);
}

// (cos, sin) of rotation pairs 2j and 2j + 1 of one row is base[j * stride]: from the
// position table at the row's position (pos given), or, with pos == nullptr, from the
// per-row table of tg_rope_rows (block j of consecutive rows contiguous, row stride
// max_pos), where a warp's loads of one block are contiguous.
struct RopeRow {
  const float4* base;
  int64_t stride;
};
__device__ __forceinline__ RopeRow rope_row(const GemmParams& p, int64_t grow, int pos) {
  const float4* t = reinterpret_cast<const float4*>(p.cos_sin);
  if (p.pos) return {t + (int64_t)pos * 32, 1};
  return {t + (grow < p.M ? grow : 0), (int64_t)p.max_pos};
}

// Epilogue of one output row held by this thread: BN accumulator columns at TMEM
// address `tbase` (the warp's lane quarter), output columns n0 .. n0 + BN.  All lanes
// of the warp must call it (tcgen05.ld is warp-collective).  Returns the row's score
// for EpiScore.
template <int BN, int EPI>
__device__ __forceinline__ float epilogue_row(const GemmParams& p, uint32_t tbase, int64_t grow,
                                              int n0, float rscale, const float* w2s) {
  const bool live = grow < p.M;
  float score = 0.f;
  if (EPI == EpiQKV) {
    // destination of this tile: Q, K or V (tiles never straddle the boundaries)
    uint16_t* dst;
    int dcol;
    if (n0 < p.q_cols) {
      dst = p.c + grow * p.ldc;
      dcol = n0;
    } else if (n0 < p.q_cols + p.k_cols) {
      dst = p.k_out + grow * p.ld_kv;
      dcol = n0 - p.q_cols;
    } else {
      dst = p.v_out + grow * p.ld_kv;
      dcol = n0 - p.q_cols - p.k_cols;
    }
    const bool rope = n0 < p.q_cols + p.k_cols;
    int pos = (rope && live && p.pos) ? p.pos[grow] : 0;
    if (p.pos && (pos < 0 || pos >= p.max_pos)) {
      if (live && p.status) atomicOr(p.status, TG_STATUS_BOUNDS);
      pos = 0;
    }
    const RopeRow rr = rope_row(p, grow, pos);
#pragma unroll 1
    for (int pr = 0; pr < BN / 64; ++pr) {
      // chunk pairs (0,2), (1,3), (4,6), (5,7): columns i and i + 64 of one head
      const int ca = (pr & 1) + 4 * (pr >> 1), cb = ca + 2;
      uint32_t ra[32], rb[32];
      tmem_ld32(tbase + ca * 32, ra);
      tmem_ld32(tbase + cb * 32, rb);
      tmem_wait_ld();
      if (live) {
        uint4* da = reinterpret_cast<uint4*>(dst + dcol + ca * 32);
        uint4* db = reinterpret_cast<uint4*>(dst + dcol + cb * 32);
        const float4* cs = rr.base + (ca & 3) * 16 * rr.stride;  // pairs i = (ca&3)*32 ..
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t wa[4], wb[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = u * 8 + 2 * e;
            float x1a = __uint_as_float(ra[i]) * rscale, x1b = __uint_as_float(ra[i + 1]) * rscale;
            float x2a = __uint_as_float(rb[i]) * rscale, x2b = __uint_as_float(rb[i + 1]) * rscale;
            if (rope) {
              const float4 t = cs[(i >> 1) * rr.stride];  // (cos_i, sin_i, cos_i+1, sin_i+1)
              const float y1a = x1a * t.x - x2a * t.y, y2a = x2a * t.x + x1a * t.y;
              const float y1b = x1b * t.z - x2b * t.w, y2b = x2b * t.z + x1b * t.w;
              x1a = y1a;
              x2a = y2a;
              x1b = y1b;
              x2b = y2b;
            }
            wa[e] = pack_bf16x2(x1a, x1b);
            wb[e] = pack_bf16x2(x2a, x2b);
          }
          da[u] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          db[u] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
        }
      }
    }
    return 0.f;
  }
  float ssq = 0.f;
#pragma unroll 1
  for (int c = 0; c < BN / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(tbase + c * 32, r);
    tmem_wait_ld();
    if (EPI == EpiStore) {
      if (live) {
        const int col = n0 + c * 32;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * rscale;
        if (p.residual) {
          const uint4* rp = reinterpret_cast<const uint4*>(p.residual + grow * p.ldr + col);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 t = rp[u];
            const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = unpack_bf16x2(w[e]);
              v[u * 8 + 2 * e] += f.x;
              v[u * 8 + 2 * e + 1] += f.y;
            }
          }
        }
        uint4* cp = reinterpret_cast<uint4*>(p.c + grow * p.ldc + col);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            w[e] = pack_bf16x2(v[u * 8 + 2 * e], v[u * 8 + 2 * e + 1]);
            if (p.row_ssq_out) {  // sums of squares of the values as stored (bf16)
              const float2 f = unpack_bf16x2(w[e]);
              ssq = fmaf(f.x, f.x, ssq);
              ssq = fmaf(f.y, f.y, ssq);
            }
          }
          cp[u] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        if (p.row_ssq_out && (c & 3) == 3) {
          p.row_ssq_out[grow * p.ld_ssq_out + (n0 + c * 32) / 128] = ssq;
          ssq = 0.f;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float u = __uint_as_float(r[i]) * rscale;
        score = fmaf(w2s[c * 32 + i], u / (1.0f + __expf(-u)), score);
      }
    }
  }
  return score;
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(192, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                GemmParams p) {
  using Cfg = GemmCfg<BN, STAGES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* tiles = smem;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::TILE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* w2s = reinterpret_cast<float*>(smem + Cfg::TILE_BYTES + Cfg::BAR_BYTES);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t m0 = (int64_t)blockIdx.x * Cfg::BM;
  const int n0 = blockIdx.y * BN;
  const int nk = p.K / Cfg::BK;
  const bool norm_here = p.rmsnorm && !p.row_ssq_in;  // epilogue warps consume A stages

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + (norm_here ? 128 : 0));  // MMA commit + each norm reader
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
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  griddep_wait();  // operands and outputs may belong to earlier grids
  if (EPI == EpiScore) {
    for (int i = tid; i < BN; i += Cfg::THREADS) w2s[i] = p.w2[n0 + i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, p.status)) break;
        unsigned char* a_s = tiles + s * Cfg::STAGE_BYTES;
        mbar_arrive_expect_tx(&full[s], Cfg::STAGE_BYTES);
        tma_load_2d(a_s, &tmA, kb * Cfg::BK, (int32_t)m0, &full[s]);
        tma_load_2d(a_s + Cfg::A_BYTES, &tmB, kb * Cfg::BK, n0, &full[s]);
        ++issued;
      }
      // Never leave the CTA with bulk copies still landing in its shared memory.
      for (int kb = issued - STAGES < 0 ? 0 : issued - STAGES; kb < issued; ++kb)
        mbar_wait(&full[kb % STAGES], (uint32_t)(kb / STAGES) & 1u, nullptr, p.status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!mbar_wait(&full[s], ph, abort_flag, p.status)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(tiles + s * Cfg::STAGE_BYTES);
        const uint32_t b_addr = a_addr + Cfg::A_BYTES;
#pragma unroll
        for (int k = 0; k < Cfg::BK / 16; ++k) {
          const uint64_t ad = sw128_desc(a_addr + k * 32, 16, 1024);
          const uint64_t bd = sw128_desc(b_addr + k * 32, 16, 1024);
          mma_ss(tmem, ad, bd, idesc, (kb | k) != 0);
        }
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
    float ss = 0.f;
    if (norm_here) {
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % STAGES;
        const uint32_t ph = (uint32_t)(kb / STAGES) & 1u;
        if (!warp_all(mbar_wait(&full[s], ph, abort_flag, p.status))) break;
        const unsigned char* rowp = tiles + s * Cfg::STAGE_BYTES + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // the row's 16-byte chunks in any order cover the whole row; XOR-ing the
          // chunk index with the row keeps each quarter-warp on distinct banks
          const uint4 v = *reinterpret_cast<const uint4*>(rowp + ((j ^ (row & 7)) << 4));
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = unpack_bf16x2(w[e]);
            ss = fmaf(f.x, f.x, ss);
            ss = fmaf(f.y, f.y, ss);
          }
        }
        // Every reading thread releases the stage itself: its arrive (release) orders
        // its own shared-memory reads before the stage is handed back, and the proxy
        // fence orders them before the TMA write that refills it.  A single arrive by
        // lane 0 after __syncwarp did not order the other lanes' reads, and refills
        // were seen to overwrite rows still being read (rows with a wrong RMS).
        fence_proxy_async_smem();
        mbar_arrive(&empty[s]);
      }
    }
    float rscale = 1.0f;
    if (p.rmsnorm) {
      if (p.row_ssq_in) rscale = grow < p.M ? rscale_from_ssq(p, grow) : 1.0f;
      else rscale = rsqrtf(ss / (float)p.K + p.eps);
    }
    const bool ok = warp_all(mbar_wait(acc_full, 0, abort_flag, p.status));
    tc_fence_after();
    if (ok) {
      const uint32_t tbase = tmem + ((uint32_t)(q * 32) << 16);
      const float score = epilogue_row<BN, EPI>(p, tbase, grow, n0, rscale, w2s);
      if (EPI == EpiScore) {
        if (grow < p.M) p.s_out[grow] = score;
        float sq = grow < p.M ? score * score : 0.f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xFFFFFFFFu, sq, o);
        if (lane == 0 && m0 + q * 32 < p.M) p.partial[(m0 + q * 32) >> 5] = sq;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

// ------------------------------------------------------------------ CTA-pair kernel

// Tensor maps of the CTA-pair kernel (boxes of 64 columns x 128 rows, 128-byte swizzle).
struct PairMaps {
  CUtensorMap a, b;    // operands A [M, K] and W [N, K]
  CUtensorMap out[3];  // EpiStore: out[0] = C [M, N]; EpiQKV: Q [M, q_cols], K rows, V rows
  CUtensorMap res;     // EpiStore with a residual: R [M, N]
};

template <int STAGES>
struct PairCfg {
  static constexpr int BM = 128, BN = 256, BK = 64;   // per CTA: 128 rows of A, 128 of W
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = (BN / 2) * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TILE_BYTES = STAGES * STAGE_BYTES;
  static constexpr int BOX_BYTES = BM * 64 * 2;        // one 64-column box of the output tile
  static constexpr int OUT_BYTES = 4 * BOX_BYTES;      // staging of one 128 x 256 output tile
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM = 1024 + TILE_BYTES + OUT_BYTES + BAR_BYTES;
  static constexpr int THREADS = 384;                  // three warpgroups
  // Registers per thread after setmaxnreg: warpgroup 0 (producer, MMA issuer and two
  // idle warps) gives up what the epilogue warpgroups take.  The split needs a launch
  // allocation of at least (128 * LOW + 256 * HIGH) / 384 = 160 registers per thread.
  static constexpr int REGS_LOW = 80, REGS_HIGH = 200;
  static constexpr int REGS_LAUNCH_MIN = (128 * REGS_LOW + 256 * REGS_HIGH) / 384;
  static constexpr int TMEM_COLS = 2 * BN;             // two accumulators (double buffer)
};

// Byte offset of 16-byte chunk k (columns 8k .. 8k + 7) of row r inside a box of 64 bf16
// columns stored with the 128-byte swizzle: the chunk index is XOR-ed with r mod 8.
__device__ __forceinline__ uint32_t sw128_chunk(int r, int k) {
  return (uint32_t)(r * 128 + ((k ^ (r & 7)) << 4));
}

// Stream-K fixup: add the other pieces' fp32 partial sums (in k order) to 32 accumulator
// columns just read from TMEM; `chunk` is the 32-column piece within the epilogue group's
// 128 columns, adds[k] already points at this thread's row.
template <int MAXADD>
__device__ __forceinline__ void add_partials(uint32_t (&r)[32], int chunk,
                                             const float4* const (&adds)[MAXADD], int n_add) {
#pragma unroll
  for (int k = 0; k < MAXADD; ++k) {
    if (k < n_add) {
      const float4* pp = adds[k] + chunk * 8 * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float4 v = __ldcg(pp + u * 128);
        r[4 * u] = __float_as_uint(__uint_as_float(r[4 * u]) + v.x);
        r[4 * u + 1] = __float_as_uint(__uint_as_float(r[4 * u + 1]) + v.y);
        r[4 * u + 2] = __float_as_uint(__uint_as_float(r[4 * u + 2]) + v.z);
        r[4 * u + 3] = __float_as_uint(__uint_as_float(r[4 * u + 3]) + v.w);
      }
    }
  }
}

// Per-row inputs of the pair epilogue that do not depend on the accumulator; the
// epilogue warps read them while the tile's MMAs run.
__device__ __forceinline__ float pair_row_rscale(const GemmParams& p, int64_t grow) {
  return (p.rmsnorm && p.row_ssq_in && grow < p.M) ? rscale_from_ssq(p, grow) : 1.0f;
}
template <int EPI>
__device__ __forceinline__ int pair_row_pos(const GemmParams& p, int64_t grow, int n0) {
  if (EPI != EpiQKV && EPI != EpiQKVNorm) return 0;
  const bool live = grow < p.M;
  if (!p.pos) return 0;  // per-row table: no position lookup
  int pos = (live && n0 < p.q_cols + p.k_cols) ? p.pos[grow] : 0;
  if (pos < 0 || pos >= p.max_pos) {
    if (live && p.status) atomicOr(p.status, TG_STATUS_BOUNDS);
    pos = 0;
  }
  return pos;
}

// The 16 (cos, sin) blocks (32 rotation pairs) of one half of a RoPE head, from block j0.
__device__ __forceinline__ void pair_rope_load(const RopeRow& rr, int j0, float4 (&rt)[16]) {
#pragma unroll
  for (int j = 0; j < 16; ++j) rt[j] = rr.base[(int64_t)(j0 + j) * rr.stride];
}
// Before the accumulator wait: the first half's blocks of a RoPE tile (Q or K columns of
// the QKV epilogues), whose latency then hides under the tile's MMAs.
template <int EPI>
__device__ __forceinline__ void pair_rope_prefetch(const GemmParams& p, int64_t grow, int n0,
                                                   int pos, float4 (&rt)[16]) {
  if ((EPI == EpiQKV || EPI == EpiQKVNorm) && n0 < p.q_cols + p.k_cols)
    pair_rope_load(rope_row(p, grow, pos), 0, rt);
}

// Columns [128 h, 128 h + 128) of one 256 x 256 output tile of the pair (each CTA: 128
// rows, staged in shared memory as four swizzled 64-column boxes); `row` is the thread's
// row in the CTA's half, `tacc` the TMEM address of the row's accumulator (lane quarter
// and buffer included); `rscale` and `pos` come from pair_row_rscale / pair_row_pos.
template <int EPI, int MAXADD>
__device__ __forceinline__ void pair_epilogue_half(const GemmParams& p, unsigned char* out_s,
                                                   uint32_t tacc, int row, int64_t grow, int n0,
                                                   int h, bool has_res, float rscale, int pos,
                                                   float4 (&rt)[16],
                                                   const float4* const (&adds)[MAXADD],
                                                   int n_add) {
  const bool live = grow < p.M;
  if (EPI == EpiQKV || EPI == EpiQKVNorm) {
    const bool rope = n0 < p.q_cols + p.k_cols;
    // QK-norm: this group's 128 columns are one Q or K head of the row; a first pass
    // over them gives the head's RMS
    float qk = 1.f;
    const float* nw = nullptr;
    if (EPI == EpiQKVNorm && rope) {
      nw = n0 < p.q_cols ? p.q_norm_w : p.k_norm_w;
      float ss = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tacc + (4 * h + c) * 32, r);
        tmem_wait_ld();
        add_partials(r, c, adds, n_add);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float v = __uint_as_float(r[i]);
          ss = fmaf(v, v, ss);
        }
      }
      qk = rsqrtf(ss * rscale * rscale * (1.0f / 128.0f) + p.qk_eps);
    }
    const float scale = rscale * qk;
    const RopeRow rr = rope_row(p, grow, pos);
#pragma unroll 1
    for (int pr = 0; pr < 2; ++pr) {
      // 32-column pieces ca and ca + 2 hold columns i and i + 64 of one 128-column head
      const int ca = 4 * h + pr, cb = ca + 2;
      // (cos, sin) blocks of this half: the first half's were loaded while the tile's
      // MMAs ran (pair_rope_prefetch); the second half's are requested here together,
      // ahead of the TMEM loads
      if (rope && pr == 1) pair_rope_load(rr, 16, rt);
      uint32_t ra[32], rb[32];
      tmem_ld32(tacc + ca * 32, ra);
      tmem_ld32(tacc + cb * 32, rb);
      tmem_wait_ld();
      add_partials(ra, pr, adds, n_add);
      add_partials(rb, pr + 2, adds, n_add);
      unsigned char* box_a = out_s + (ca >> 1) * PairCfg<1>::BOX_BYTES;
      unsigned char* box_b = out_s + (cb >> 1) * PairCfg<1>::BOX_BYTES;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t wa[4], wb[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = u * 8 + 2 * e;
          float x1a = __uint_as_float(ra[i]) * scale, x1b = __uint_as_float(ra[i + 1]) * scale;
          float x2a = __uint_as_float(rb[i]) * scale, x2b = __uint_as_float(rb[i + 1]) * scale;
          if (EPI == EpiQKVNorm && nw) {  // head columns c and c + 64, c = 32 pr + i
            const int c = 32 * pr + i;
            x1a *= __ldg(nw + c);
            x1b *= __ldg(nw + c + 1);
            x2a *= __ldg(nw + c + 64);
            x2b *= __ldg(nw + c + 65);
          }
          if (rope) {
            const float4 t = rt[i >> 1];  // (cos_i, sin_i, cos_i+1, sin_i+1), i in the half
            const float y1a = x1a * t.x - x2a * t.y, y2a = x2a * t.x + x1a * t.y;
            const float y1b = x1b * t.z - x2b * t.w, y2b = x2b * t.z + x1b * t.w;
            x1a = y1a;
            x2a = y2a;
            x1b = y1b;
            x2b = y2b;
          }
          wa[e] = pack_bf16x2(x1a, x1b);
          wb[e] = pack_bf16x2(x2a, x2b);
        }
        const int k = (ca & 1) * 4 + u;  // chunk of the piece within its box
        *reinterpret_cast<uint4*>(box_a + sw128_chunk(row, k)) =
            make_uint4(wa[0], wa[1], wa[2], wa[3]);
        *reinterpret_cast<uint4*>(box_b + sw128_chunk(row, k)) =
            make_uint4(wb[0], wb[1], wb[2], wb[3]);
      }
    }
    return;
  }
  if (EPI == EpiSwiGLU) {
    // Group h's 128 tile columns are 64 gate features then the same 64 up features
    // (weight rows interleaved in blocks of 64); out = SiLU(gate) * up, 64 bf16 columns
    // staged in box h.
    unsigned char* box = out_s + h * PairCfg<1>::BOX_BYTES;
#pragma unroll 1
    for (int c = 0; c < 2; ++c) {
      uint32_t rg[32], ru[32];
      tmem_ld32(tacc + 128 * h + 32 * c, rg);
      tmem_ld32(tacc + 128 * h + 64 + 32 * c, ru);
      tmem_wait_ld();
      add_partials(rg, c, adds, n_add);
      add_partials(ru, c + 2, adds, n_add);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = u * 8 + 2 * e;
          const float ga = __uint_as_float(rg[i]) * rscale, gb = __uint_as_float(rg[i + 1]) * rscale;
          const float ua = __uint_as_float(ru[i]) * rscale, ub = __uint_as_float(ru[i + 1]) * rscale;
          w[e] = pack_bf16x2(ga / (1.0f + __expf(-ga)) * ua, gb / (1.0f + __expf(-gb)) * ub);
        }
        *reinterpret_cast<uint4*>(box + sw128_chunk(row, 4 * c + u)) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    return;
  }
  float ssq = 0.f;
#pragma unroll 1
  for (int j = 2 * h; j < 2 * h + 2; ++j) {  // box j: tile columns 64 j .. 64 j + 63
    uint32_t ra[32], rb[32];
    tmem_ld32(tacc + j * 64, ra);
    tmem_ld32(tacc + j * 64 + 32, rb);
    tmem_wait_ld();
    add_partials(ra, 2 * (j - 2 * h), adds, n_add);
    add_partials(rb, 2 * (j - 2 * h) + 1, adds, n_add);
    unsigned char* box = out_s + j * PairCfg<1>::BOX_BYTES;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint4* cp = reinterpret_cast<uint4*>(box + sw128_chunk(row, k));
      float v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        v[e] = __uint_as_float(k < 4 ? ra[8 * k + e] : rb[8 * (k - 4) + e]) * rscale;
      if (has_res) {
        const uint4 t = *cp;
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = unpack_bf16x2(w[e]);
          v[2 * e] += f.x;
          v[2 * e + 1] += f.y;
        }
      }
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        w[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
        if (p.row_ssq_out) {  // sums of squares of the values as stored (bf16)
          const float2 f = unpack_bf16x2(w[e]);
          ssq = fmaf(f.x, f.x, ssq);
          ssq = fmaf(f.y, f.y, ssq);
        }
      }
      *cp = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (p.row_ssq_out && (j & 1) && live) p.row_ssq_out[grow * p.ld_ssq_out + n0 / 128 + h] = ssq;
  }
}

// One GEMM for the CTA-pair kernel: tensor maps and parameters.
struct PairJob {
  PairMaps maps;
  GemmParams p;
};

// Optional ordering between the two jobs of one launch: job 1 reads (as A and through
// row_ssq_in) the rows job 0 writes.  ready[rp] counts job 0's finished epilogue groups
// of row pair rp (each 256 x 256 tile contributes 4: two groups in each CTA); a job-1
// tile of rp starts loading once ready[rp] == target.  consumed[rp] counts job-1
// producers that passed that wait; the last one resets both, so the counters start and
// end every launch at zero (the caller zero-fills them once).
struct PairChain {
  int* ready;
  int* consumed;
  int target;
};

// Stream-K tail of a single-job launch.  The first dp_tiles tiles (whole rounds of the
// clusters) run whole, tile t on cluster t mod C; the k-blocks of the remaining tiles are
// shared out evenly, in tile order, as one contiguous range of tail_units per cluster
// ("pieces").  A piece holding a tile's first k-block finishes that tile: it runs last
// in its cluster, waits for the tile's other pieces (each the first piece of a later
// cluster's range, run before that cluster's whole tiles), adds their fp32 partial sums
// in k order to its own accumulator and runs the epilogue; the other pieces only
// publish their partial sums.
// A cluster has at most one such contributing piece, so partials and ready flags are
// indexed by cluster: part[((c * 2 + rank) * 2 + group) * 32 * 128 + f * 128 + row]
// (float4, f = 4-column group within the epilogue group's 128 columns) and
// flag[(c * 2 + rank) * 2 + group].  Every cluster must be resident at once: the launch
// is cooperative.  part == nullptr: no split.
struct PairSplit {
  float4* part;
  int* flag;
  int dp_tiles;
  int64_t tail_units;
};
constexpr int kMaxPieces = 8;  // pieces per split tile (the host keeps ranges long enough)

struct Piece {
  int t, kb0, kb1;
  int kind;  // 0: whole tile, 1: finisher (first k-blocks), 2: contributor
};

// The pieces of cluster c in the order the cluster runs them (SPLIT = false: the plain
// tile loop, everything below it compiled out): a tail range that starts
// inside a tile begins with a contributing piece, which runs first (its partial sums are
// then published before the cluster's first epilogue, and the finisher that waits for
// them does not wait behind that epilogue); then the whole tiles; then the rest of the
// range, whose last piece may be a finisher.
template <bool SPLIT>
struct PieceIter {
  int c, C, n_tiles, nk, dp_tiles;
  int64_t u, u1;
  int i;
  bool split, lead_done;
  __device__ PieceIter(int c_, int C_, int n_tiles_, int nk_, const PairSplit& sp)
      : c(c_), C(C_), n_tiles(n_tiles_), nk(nk_), dp_tiles(0), u(0), u1(0), i(0),
        split(SPLIT && sp.part != nullptr), lead_done(false) {
    if (SPLIT && split) {
      dp_tiles = sp.dp_tiles;
      u = sp.tail_units * c / C;
      u1 = sp.tail_units * (c + 1) / C;
    }
  }
  __device__ bool tail_piece(Piece& pc) {
    const int tt = (int)(u / nk);
    const int kb0 = (int)(u % nk);
    const int64_t left = u1 - u;
    const int kb1 = left < (int64_t)(nk - kb0) ? kb0 + (int)left : nk;
    pc = {dp_tiles + tt, kb0, kb1, kb0 == 0 ? (kb1 == nk ? 0 : 1) : 2};
    u += kb1 - kb0;
    return true;
  }
  __device__ bool next(Piece& pc) {
    if (SPLIT && split && !lead_done) {
      lead_done = true;
      if (u < u1 && u % nk != 0) return tail_piece(pc);
    }
    const int t = c + i * C;
    if (!(SPLIT && split) ? t < n_tiles : t < dp_tiles) {
      pc = {t, 0, nk, 0};
      ++i;
      return true;
    }
    if (!(SPLIT && split) || u >= u1) return false;
    return tail_piece(pc);
  }
};

// Persistent CTA-pair GEMM: each cluster of two CTAs walks the 256 x 256 output tiles
// t = cluster, cluster + clusters, ... of job 0 and then of job 1 (tiles of job 1 follow
// all of job 0's in that order, so a job-1 tile only ever waits for job-0 tiles that
// are already running or done).  Roles per CTA:
//   warp 0     one thread streams A and W k-blocks of every tile through the ring;
//   warp 1     TMEM owner; in the even CTA one thread issues the M=256 MMAs into
//              accumulator buffer (tile index & 1);
//   warps 2-3  idle (warpgroup 0 lowers its registers for the epilogue warpgroups);
//   warps 4-11 epilogue of the previous tile while the next one accumulates, as two
//              independent groups of four warps (one per TMEM lane quarter, one per
//              warpgroup), group g owning tile columns [128 g, 128 g + 128): TMEM ->
//              registers -> bf16 in swizzled staging boxes -> TMA stores.  For EpiStore
//              with a residual, the group's boxes are first filled with the residual
//              rows by a TMA load issued one tile ahead; a RoPE head's first (cos, sin)
//              blocks are loaded before the accumulator wait.
// Barriers: full/empty per ring stage (full lives in the even CTA and counts both CTAs'
// bytes); acc_full[b] (the even CTA's commit, in both CTAs); acc_empty[b] (even CTA,
// one arrive per epilogue group of each CTA once it has read buffer b); res_full[g].
template <int STAGES, int EPI0, int EPI1, bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    gemm_pair_kernel(const __grid_constant__ PairJob job0, const __grid_constant__ PairJob job1,
                     PairChain chain, PairSplit split) {
  using Cfg = PairCfg<STAGES>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* tiles = smem;
  unsigned char* out_s = smem + Cfg::TILE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(out_s + Cfg::OUT_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;   // [2]
  uint64_t* acc_empty = acc_full + 2;    // [2]
  uint64_t* res_full = acc_empty + 2;   // [2]
  uint64_t* drain = res_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int cluster = (int)(blockIdx.x >> 1), n_clusters = (int)(gridDim.x >> 1);
  const int tn0 = job0.p.N / Cfg::BN, tn1 = job1.p.M > 0 ? job1.p.N / Cfg::BN : 1;
  const int n_tiles0 = (int)((job0.p.M + 255) / 256) * tn0;
  const int n_tiles1 = job1.p.M > 0 ? (int)((job1.p.M + 255) / 256) * tn1 : 0;
  const int n_tiles = n_tiles0 + n_tiles1;
  uint32_t* status = job0.p.status;
  // tile t -> job, row pair and first column of the tile
  auto decode = [&](int t, int& job, int& rp, int& n0) {
    job = t >= n_tiles0;
    const int u = job ? t - n_tiles0 : t;
    const int tn = job ? tn1 : tn0;
    rp = u / tn;
    n0 = (u % tn) * Cfg::BN;
  };
  auto has_res = [&](int job) {
    return job ? (EPI1 == EpiStore && job1.p.residual != nullptr)
               : (EPI0 == EpiStore && job0.p.residual != nullptr);
  };

  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
      mbar_init(&res_full[b], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&job0.maps.a);
    tma_prefetch_desc(&job0.maps.b);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Past the previous grid: the next one may be scheduled on the SMs this grid leaves
  // free (all of its clusters are resident, one wave), to wait there for its completion.
  griddep_wait();
  griddep_launch_dependents();
  if (warp < 4) {
    regs_dec<Cfg::REGS_LOW>();  // warpgroup 0: producer, MMA issuer, two idle warps
    if (warp == 0) {
      if (lane == 0) {
        // The odd CTA's bytes may reach the even CTA's barrier before the even CTA's
        // expect_tx: the phase cannot complete early, as it still waits for that arrive.
        // A stage is reloaded only after the even CTA's commit freed it, which follows
        // the completion of that barrier's previous phase.
        const uint32_t full_lead0 = mapa_shared(smem_u32(&full[0]), 0);
        griddep_wait();
        int kg = 0;
        bool ok = true;
        PieceIter<SPLIT> pit(cluster, n_clusters, n_tiles, job0.p.K / Cfg::BK, split);
        Piece pc;
        while (ok && pit.next(pc)) {
          const int t = pc.t;
          int job, rp, n0;
          decode(t, job, rp, n0);
          const PairJob& jb = job ? job1 : job0;
          if (job && chain.ready) {
            // job 0 must have finished every column of these rows
            if (!wait_count_gpu(chain.ready + rp, chain.target, abort_flag, status)) break;
            fence_proxy_async_global();  // the rows are read by TMA next
            if (atomicAdd(chain.consumed + rp, 1) == 2 * tn1 - 1) {
              chain.ready[rp] = 0;  // every producer of these rows has passed its wait
              chain.consumed[rp] = 0;
            }
          }
          const int64_t m0 = (int64_t)rp * 256 + rank * 128;
          const int nb = n0 + (int)rank * (Cfg::BN / 2);
          const int nk = jb.p.K / Cfg::BK;
          const int kb_end = job ? nk : pc.kb1;
          for (int kb = job ? 0 : pc.kb0; kb < kb_end; ++kb, ++kg) {
            const int s = kg % STAGES;
            const uint32_t ph = (uint32_t)(kg / STAGES) & 1u;
            if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, status)) {
              ok = false;
              break;
            }
            unsigned char* a_s = tiles + s * Cfg::STAGE_BYTES;
            if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * Cfg::STAGE_BYTES);
            tma_load_2d_pair(a_s, &jb.maps.a, kb * Cfg::BK, (int32_t)m0, full_lead0 + s * 8);
            tma_load_2d_pair(a_s + Cfg::A_BYTES, &jb.maps.b, kb * Cfg::BK, nb, full_lead0 + s * 8);
          }
        }
        // The even CTA waits until the last stages' bytes (both CTAs') have landed; the odd
        // CTA is held by the closing cluster barrier until then.
        if (rank == 0)
          for (int g = kg - STAGES < 0 ? 0 : kg - STAGES; g < kg; ++g)
            mbar_wait(&full[g % STAGES], (uint32_t)(g / STAGES) & 1u, nullptr, status);
      }
    } else if (warp == 1) {
      if (lane == 0 && rank == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(256, Cfg::BN, false, false);
        const uint32_t empty_peer0 = mapa_shared(smem_u32(&empty[0]), 1);
        const uint32_t acc_full_peer0 = mapa_shared(smem_u32(&acc_full[0]), 1);
        int kg = 0, i = 0;
        bool ok = true;
        PieceIter<SPLIT> pit(cluster, n_clusters, n_tiles, job0.p.K / Cfg::BK, split);
        Piece pc;
        for (; ok && pit.next(pc); ++i) {
          const int t = pc.t;
          const int b = i & 1;
          const bool j1 = t >= n_tiles0;
          const int kb_begin = j1 ? 0 : pc.kb0;
          const int kb_end = j1 ? job1.p.K / Cfg::BK : pc.kb1;
          // both CTAs' epilogues are done with this buffer (first use passes at once)
          if (!mbar_wait(&acc_empty[b], ((uint32_t)(i >> 1) & 1u) ^ 1u, abort_flag, status)) break;
          tc_fence_after();
          const uint32_t d = tmem + (uint32_t)(b * Cfg::BN);
          for (int kb = kb_begin; kb < kb_end; ++kb, ++kg) {
            const int s = kg % STAGES;
            const uint32_t ph = (uint32_t)(kg / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph, abort_flag, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(tiles + s * Cfg::STAGE_BYTES);
            const uint32_t b_addr = a_addr + Cfg::A_BYTES;
  #pragma unroll
            for (int k = 0; k < Cfg::BK / 16; ++k)
              mma_ss_pair(d, sw128_desc(a_addr + k * 32, 16, 1024),
                          sw128_desc(b_addr + k * 32, 16, 1024), idesc,
                          (kb != kb_begin || k != 0) ? 1u : 0u);
            mma_commit_pair(smem_u32(&empty[s]));
            mma_commit_pair(empty_peer0 + s * 8);
          }
          if (!ok) break;
          mma_commit_pair(smem_u32(&acc_full[b]));
          mma_commit_pair(acc_full_peer0 + b * 8);
        }
        mma_commit_pair(smem_u32(drain));
        mbar_wait(drain, 0, nullptr, status);  // all MMAs (and their arrives) done
      }
    }
  } else {
    regs_inc<Cfg::REGS_HIGH>();  // the two epilogue warpgroups
    const int q = warp & 3;        // TMEM lane quarter this warp may access
    const int g = (warp - 4) >> 2;  // epilogue group: tile columns [128 g, 128 g + 128)
    const int row = q * 32 + lane;
    const bool elected = (warp & 3) == 0 && lane == 0;  // warps 4 and 8
    const uint32_t bar_id = 1 + (uint32_t)g;
    const uint32_t acc_empty_lead0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    griddep_wait();
    int res_loads = 0;  // residual half-tiles requested by this group's elected thread
    auto load_res = [&](int t) {
      int job, rp, n0;
      decode(t, job, rp, n0);
      const PairJob& jb = job ? job1 : job0;
      const int64_t m0 = (int64_t)rp * 256 + rank * 128;
      ++res_loads;
      mbar_arrive_expect_tx(&res_full[g], 2 * Cfg::BOX_BYTES);
      for (int j = 2 * g; j < 2 * g + 2; ++j)
        tma_load_2d(out_s + j * Cfg::BOX_BYTES, &jb.maps.res, n0 + 64 * j, (int32_t)m0,
                    &res_full[g]);
    };
    auto res_of = [&](int t) {
      int job, rp, n0;
      decode(t, job, rp, n0);
      return has_res(job);
    };
    PieceIter<SPLIT> pit(cluster, n_clusters, n_tiles, job0.p.K / Cfg::BK, split);
    PieceIter<SPLIT> peek = pit;  // one piece ahead: the residual of the next piece loads early
    Piece pc, nx;
    bool has_next = peek.next(nx);
    auto needs_res = [&](const Piece& q) { return q.kind != 2 && res_of(q.t); };
    if (elected && has_next && needs_res(nx)) load_res(nx.t);
    const int nk0 = job0.p.K / Cfg::BK;
    int i = 0, res_used = 0;
    for (; pit.next(pc); ++i) {
      has_next = peek.next(nx);  // nx: the piece after pc
      const int t = pc.t;
      const int b = i & 1;
      int job, rp, n0;
      decode(t, job, rp, n0);
      const PairJob& jb = job ? job1 : job0;
      const bool with_res = pc.kind != 2 && has_res(job);
      const int64_t m0 = (int64_t)rp * 256 + rank * 128;
      // job 1 of a chain reads job 0's row sums of squares only after the wait below
      const bool late_ssq = job && chain.ready;
      float rscale = (pc.kind != 2 && !late_ssq) ? pair_row_rscale(jb.p, m0 + row) : 1.0f;
      const int pos = pc.kind == 2 ? 0
                      : job        ? pair_row_pos<EPI1>(jb.p, m0 + row, n0)
                                   : pair_row_pos<EPI0>(jb.p, m0 + row, n0);
      float4 rt[16];  // first half of a RoPE head's (cos, sin) blocks
      if (pc.kind != 2) {
        if (job)
          pair_rope_prefetch<EPI1>(jb.p, m0 + row, n0, pos, rt);
        else
          pair_rope_prefetch<EPI0>(jb.p, m0 + row, n0, pos, rt);
      }
      bool ok = mbar_wait(&acc_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, status);
      if (ok && with_res) ok = mbar_wait(&res_full[g], (uint32_t)res_used & 1u, abort_flag, status);
      if (with_res) ++res_used;
      // a finisher adds the partial sums of the tile's other pieces: the clusters whose
      // tail ranges start inside this tile, in k order
      constexpr int kAdd = SPLIT ? kMaxPieces : 1;
      const float4* adds[kAdd];
      int add_cl[kAdd];
      int n_add = 0;
      if (SPLIT && pc.kind == 1) {
        const int64_t lo = (int64_t)(t - split.dp_tiles) * nk0, hi = lo + nk0;
        for (int c2 = cluster + 1; c2 < n_clusters && n_add < kAdd; ++c2) {
          const int64_t b2 = split.tail_units * c2 / n_clusters;
          if (b2 >= hi) break;
          if (b2 > lo) {
            add_cl[n_add] = c2;
            adds[n_add++] = split.part + (int64_t)((c2 * 2 + (int)rank) * 2 + g) * 32 * 128 + row;
          }
        }
        if (elected)
          for (int k = 0; k < n_add && ok; ++k)
            ok = wait_flag_gpu(split.flag + (add_cl[k] * 2 + (int)rank) * 2 + g, abort_flag, status);
      }
      // job 1 reads job 0's row sums of squares: its producer acquired job 0's release
      // before the loads behind this accumulator; a device fence orders this thread's
      // reads after it too (the counter itself may already be reset by then)
      if (late_ssq) __threadfence();
      // one decision for the group's four warps (they meet at named barriers below)
      if (!named_bar_and(bar_id, 128, ok)) break;
      tc_fence_after();
      const uint32_t tacc = tmem + (uint32_t)(b * Cfg::BN) + ((uint32_t)(q * 32) << 16);
      if (SPLIT && pc.kind == 2) {
        // contributor: the group's 128 raw accumulator columns go to this cluster's
        // partial block (float4 per 4 columns, row-contiguous: coalesced)
        float4* dst = split.part + (int64_t)((cluster * 2 + (int)rank) * 2 + g) * 32 * 128 + row;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t r[32];
          tmem_ld32(tacc + (4 * g + c) * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 8; ++u)
            dst[(c * 8 + u) * 128] =
                make_float4(__uint_as_float(r[4 * u]), __uint_as_float(r[4 * u + 1]),
                            __uint_as_float(r[4 * u + 2]), __uint_as_float(r[4 * u + 3]));
        }
        __threadfence();  // this thread's part is visible GPU-wide before the flag
        tc_fence_before();
        named_bar_sync(bar_id, 128);
        if (elected) {
          if (rank == 0)
            mbar_arrive(&acc_empty[b]);
          else
            mbar_arrive_cluster(acc_empty_lead0 + b * 8);
          st_release_gpu(split.flag + (cluster * 2 + (int)rank) * 2 + g, 1);
          if (has_next && needs_res(nx)) load_res(nx.t);
        }
        named_bar_sync(bar_id, 128);
        continue;
      }
      if (late_ssq) rscale = pair_row_rscale(jb.p, m0 + row);
      if (job)
        pair_epilogue_half<EPI1, kAdd>(jb.p, out_s, tacc, row, m0 + row, n0, g, with_res,
                                             rscale, pos, rt, adds, n_add);
      else
        pair_epilogue_half<EPI0, kAdd>(jb.p, out_s, tacc, row, m0 + row, n0, g, with_res,
                                             rscale, pos, rt, adds, n_add);
      const bool publish = !job && chain.ready;  // job 1 waits for these rows
      if (publish) __threadfence();  // row sums of squares visible before the count
      tc_fence_before();
      fence_proxy_async_smem();  // staging writes visible to the TMA stores
      named_bar_sync(bar_id, 128);
      if (elected) {
        if (rank == 0)
          mbar_arrive(&acc_empty[b]);
        else
          mbar_arrive_cluster(acc_empty_lead0 + b * 8);
        // every thread of the group has read the partials: leave the flags at zero
        for (int k = 0; k < n_add; ++k) split.flag[(add_cl[k] * 2 + (int)rank) * 2 + g] = 0;
        int mi = 0, x = n0;
        const int epi = job ? EPI1 : EPI0;
        if (epi == EpiQKV || epi == EpiQKVNorm) {
          if (n0 >= jb.p.q_cols + jb.p.k_cols) {
            mi = 2;
            x = n0 - jb.p.q_cols - jb.p.k_cols;
          } else if (n0 >= jb.p.q_cols) {
            mi = 1;
            x = n0 - jb.p.q_cols;
          }
        }
        if (epi == EpiSwiGLU)  // 64 output columns per group: features n0 / 2 + 64 g ..
          tma_store_2d(&jb.maps.out[0], n0 / 2 + 64 * g, (int32_t)m0, out_s + g * Cfg::BOX_BYTES);
        else
          for (int j = 2 * g; j < 2 * g + 2; ++j)
            tma_store_2d(&jb.maps.out[mi], x + 64 * j, (int32_t)m0, out_s + j * Cfg::BOX_BYTES);
        bulk_commit_group();
        if (publish) {
          bulk_wait_all();             // the rows are in global memory
          fence_proxy_async_global();  // ... and ordered before the release below
          atomicAdd_release_gpu(chain.ready + rp, 1);
        } else {
          bulk_wait_read_all();  // the group's staging boxes may be overwritten from here on
        }
        if (has_next && needs_res(nx)) load_res(nx.t);
      }
      named_bar_sync(bar_id, 128);
    }
    if (elected) {
      // the staging boxes are read before the CTA exits; the stores' global writes are
      // complete, like every other write of the grid, when the kernel is
      bulk_wait_read_all();
      // after an abort: a residual load may still be landing in the staging boxes
      if (res_loads > res_used)
        mbar_wait(&res_full[g], (uint32_t)(res_loads - 1) & 1u, nullptr, status);
    }
  }
  __syncwarp();  // the role branches above diverge inside warps 0 and 1
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while the pair's MMAs or arrives may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace tg
