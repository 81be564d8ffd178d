// Token-gated causal GQA flash attention on tcgen05 tensor cores.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 端到端训练的关键在 token 门控注意力 (a learnable per-head gain multiplies the importance
// score, which joins q.k/sqrt(d) in the softmax; an SSMax-style temperature rescales
// by the log-ratio of kept count to original position); "斯坦福与 UC Berkeley 提出
// TokenGate：token 门控注意力让长上下文预填充最高快 11.3 倍", section "What is token-gated
// attention?" (each kept token's score is a bias on the logits); "TokenGate：让模型学会
// 跳读，而不只压缩 KV 缓存", figure 1(c) (key bias, positive per-head gain, temperature).
// Formula implemented:
//   logit[r, c] = tau_r * q_r.k_c / sqrt(d) + gamma_h * bias_c   (c <= r, same request)
//   tau_r = beta * ln(r + 1) / ln(p_r + 1), tau_r = beta when p_r = 0.
//
// One CTA = one request, one tile of 128 query ranks, one share of its causal key range
// (split-KV, see the plan below), one kv head and the two q heads (h0, h0 + 1) that read
// it.  Tensor memory (512 columns):
//   S0/P0 [0,128)  S1/P1 [128,256)  O0 [256,384)  O1 [384,512)
// Warpgroup 0 (warps 0-3, registers lowered to 120): warp 0 loads Q once and then K/V
// tiles through a 2-stage TMA ring (a K stage is released once both heads' S MMAs have
// read it, a V stage after both PV MMAs) and writes each tile's key bias as two extra
// bf16 K columns; warp 1 issues S = Q K^T + (one more K=16 step) gain x bias, both
// operands in shared memory, and O += P V (P read from TMEM, V an MN-major shared
// operand).
// Warpgroups 1 and 2 (registers raised to 192) are the softmax of head h0 and h0 + 1,
// one thread per query row.  S from TMEM is the row's logit divided by its temperature
// factor t = tau * log2(e) / sqrt(d) (the extra MMA step adds gamma * log2(e) / t times
// the bias), so the softmax takes the row max of S, forms t * S - m with one packed
// fp32x2 FMA per two keys, exponentiates on the MUFU unit, sums in packed pairs and
// stores P to TMEM as bf16.  Masking is only applied on the diagonal tile.  The running
// max moves (and O is rescaled in TMEM) only when it grows by more than 2^8, which keeps
// P inside bf16 range.  The two heads ping-pong on the tensor core.
#include <cuda.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <functional>
#include <vector>

#include "tg_attn_common.cuh"
#include "tg_host.h"
#include "tg_ptx.cuh"

namespace tg {
namespace {

constexpr int kD = 128;         // head_dim
constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per KV tile
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 384;   // 3 warpgroups
constexpr int kLaunchRegs = 168;  // 65536 / 384, rounded down to a multiple of 8
constexpr int kRegsLow = 120;     // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsHigh = 192;    // softmax warpgroups after setmaxnreg.inc
static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
constexpr int kMaxBatch = 512;  // requests per call (tile table lives in the parameters)
constexpr int kTileBytes = kBM * kD * 2;  // 32 KB: 128 rows x 128 bf16, two 64-column boxes
constexpr float kLog2e = kAttnLog2e;
constexpr float kRescaleThreshold = 8.0f;

constexpr int kMaxParts = 8;    // parts per split query tile
constexpr int kBoxBytes = kBM * 64 * 2;  // one 64-column bf16 box of a 128-row tile
// Epilogue staging (the Q/K/V/bias region is free once every MMA has retired): a split
// part's block for both heads at 0, the bf16 output tile (2 heads x 2 boxes) after it.
constexpr int kEpiOut = 2 * (kBM * kD + 2 * kBM) * 4;

// Extra K columns of the S = Q K^T MMA that add the gate bias (layout in
// tg_attn_common.cuh).
constexpr int kExBytes = kAttnExBytes;

struct AttnSmem {
  // 1024-aligned tiles first
  static constexpr int Q0 = 0;
  static constexpr int Q1 = Q0 + kTileBytes;
  static constexpr int K = Q1 + kTileBytes;
  static constexpr int V = K + kStages * kTileBytes;
  static constexpr int AEX = V + kStages * kTileBytes;  // [head] extra A columns (gain)
  static constexpr int BEX = AEX + 2 * kExBytes;        // [stage] extra B columns (key bias)
  static constexpr int BAR = BEX + kStages * kExBytes;
  static constexpr int END = BAR + 256;
  static constexpr int BYTES = END + 1024;  // alignment slack
};

static_assert(kEpiOut % 1024 == 0 && kEpiOut + 4 * kBoxBytes <= AttnSmem::BAR,
              "epilogue staging must fit below the barriers, 1024-byte aligned");

struct AttnParams {
  const int32_t* cu_kept;
  const int32_t* kept_pos;
  const float* kept_bias;
  const float* gamma;
  float beta;
  uint16_t* o;
  int64_t ld_o;
  float* lse;
  int64_t k_total;
  int n_q_heads;
  int group;        // n_q_heads / n_kv_heads
  int head_pairs;   // group / 2
  int n_kv_heads;
  int batch;
  uint32_t* status;
  int chunk;           // key tiles per work item (split-KV); >= every request's tile count = no split
  float* part_ws;      // partial results of split query tiles (see kPartFloats), or null
  int* part_count;     // per (first item of a split tile, head group): parts arrived
  int* part_ready;     // per (work item, head group): 1 once the part's partial is written
  int32_t item_prefix[kMaxBatch + 1];  // work items before request b
};

// Floats per (work item, q head) in the split-KV workspace: 128 rows x 128 unnormalised
// O values, then 128 row maxima (log2 domain), then 128 row sums.  O is stored as 32
// groups of 4 columns, each group row-contiguous (group f of row r at float4 index
// f * 128 + r), so that one thread per row reads and writes coalesced.
constexpr int kPartFloats = kBM * kD + 2 * kBM;

__host__ __device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Work item t -> request b, query tile qt, part index and part count.  Within a request
// items run over query tiles from the heaviest (last) to the lightest, the parts of a
// tile consecutively; part i covers key tiles [i * chunk, min((i + 1) * chunk, qt + 1)).
__device__ __forceinline__ void decode_item(const AttnParams& p, int t, int& b, int& qt,
                                            int& part, int& nparts) {
  int lo = 0, hi = p.batch;  // largest b with item_prefix[b] <= t
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (p.item_prefix[mid] <= t) lo = mid; else hi = mid;
  }
  b = lo;
  int idx = t - p.item_prefix[b];
  const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
  const int ntiles = ceil_div(n_b, kBM);
  qt = ntiles - 1;
  if (p.chunk >= ntiles) {  // no split: one item per query tile
    qt = ntiles - 1 - idx;
    part = 0;
    nparts = 1;
    return;
  }
  while (true) {
    const int np = ceil_div(qt + 1, p.chunk);
    if (idx < np) {
      part = idx;
      nparts = np;
      return;
    }
    idx -= np;
    --qt;
  }
}

// Row maximum of one key tile's logits; on the diagonal tile keys past the row are set
// to -inf first.
template <bool kDiag>
__device__ __forceinline__ float row_max(uint32_t (&sv)[kBN], int rit) {
  float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
  for (int i = 0; i < kBN / 4; ++i) {
    float a = __uint_as_float(sv[4 * i]), b = __uint_as_float(sv[4 * i + 1]);
    float c = __uint_as_float(sv[4 * i + 2]), d = __uint_as_float(sv[4 * i + 3]);
    if (kDiag) {
      if (4 * i + 0 > rit) a = -INFINITY;
      if (4 * i + 1 > rit) b = -INFINITY;
      if (4 * i + 2 > rit) c = -INFINITY;
      if (4 * i + 3 > rit) d = -INFINITY;
      sv[4 * i] = __float_as_uint(a);
      sv[4 * i + 1] = __float_as_uint(b);
      sv[4 * i + 2] = __float_as_uint(c);
      sv[4 * i + 3] = __float_as_uint(d);
    }
    if (i & 1) {
      m2 = max3(m2, a, b);
      m3 = max3(m3, c, d);
    } else {
      m0 = max3(m0, a, b);
      m1 = max3(m1, c, d);
    }
  }
  return fmaxf(max3(m0, m1, m2), m3);
}

__global__ void __launch_bounds__(kThreads, 1)
    gated_attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ CUtensorMap tmO,
                           const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [kStages]
  uint64_t* v_full = k_full + kStages;     // [kStages]
  uint64_t* k_empty = v_full + kStages;    // [kStages]
  uint64_t* v_empty = k_empty + kStages;   // [kStages]
  uint64_t* bx_full = v_empty + kStages;   // [kStages] extra bias columns of the stage written
  uint64_t* ax_ready = bx_full + kStages;  // [2] the head's extra A columns written (per row)
  uint64_t* s_full = ax_ready + 2;         // [2]
  uint64_t* p_full = s_full + 2;           // [2]
  uint64_t* pv_done = p_full + 2;          // [2]
  uint64_t* p_half = pv_done + 2;          // [2] P of the tile's first 64 keys stored
  uint64_t* drain = p_half + 2;
  uint64_t* merge_full = drain + 1;        // a split tile's other part staged for the merge
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(merge_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_part = reinterpret_cast<volatile int*>(tmem_slot + 2);
  volatile int* parts_ready = reinterpret_cast<volatile int*>(tmem_slot + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&bx_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&ax_ready[h], 128);
      mbar_init(&s_full[h], 1);
      mbar_init(&p_full[h], 128);
      mbar_init(&p_half[h], 128);
      mbar_init(&pv_done[h], 1);
    }
    mbar_init(drain, 1);
    mbar_init(merge_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // everything below reads what earlier grids wrote
  griddep_wait();

  // ---- which work item: head groups vary fastest, then items heaviest first
  const int hg = p.n_kv_heads * p.head_pairs;
  const int head_grp = blockIdx.x % hg;
  const int item = blockIdx.x / hg;
  int b, qt, part, nparts;
  decode_item(p, item, b, qt, part, nparts);
  const int g = head_grp / p.head_pairs;
  const int h0 = g * p.group + 2 * (head_grp % p.head_pairs);
  const int64_t row0 = p.cu_kept[b];
  const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
  const int q0 = qt * kBM;
  // causal: key tiles 0..qt, this item's share [j0, j0 + nt)
  const int j0 = part * p.chunk;
  const int nt = min(qt + 1, j0 + p.chunk) - j0;

  if (warp < 4) {
    regs_dec<kRegsLow>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      int loaded = 0, loaded_v = 0;
      bool q_issued = false;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, 2 * kTileBytes);
        const int y = (int)(row0 + q0);
        tma_load_2d(smem + AttnSmem::Q0, &tmQ, h0 * kD, y, q_full);
        tma_load_2d(smem + AttnSmem::Q0 + kTileBytes / 2, &tmQ, h0 * kD + 64, y, q_full);
        tma_load_2d(smem + AttnSmem::Q1, &tmQ, (h0 + 1) * kD, y, q_full);
        tma_load_2d(smem + AttnSmem::Q1 + kTileBytes / 2, &tmQ, (h0 + 1) * kD + 64, y, q_full);
        q_issued = true;
      }
      // Key bias of tile j, loaded one tile ahead so its global latency overlaps the
      // wait for a free stage.
      auto load_bias = [&](int j, float (&bv)[4]) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int c = (j0 + j) * kBN + lane * 4 + e;
          bv[e] = (j < nt && c < n_b) ? p.kept_bias[row0 + c] : 0.0f;
        }
      };
      float bv[4];
      load_bias(0, bv);
      for (int j = 0; j < nt; ++j) {
        const int s = j % kStages;
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        const int y = (int)(row0 + (j0 + j) * kBN);
        // K of tile j once both heads' S MMAs of tile j - kStages are done
        if (!warp_all(mbar_wait(&k_empty[s], ph ^ 1u, abort_flag, p.status))) break;
        unsigned char* kt = smem + AttnSmem::K + s * kTileBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&k_full[s], kTileBytes);
          tma_load_2d(kt, &tmK, g * kD, y, &k_full[s]);
          tma_load_2d(kt + kTileBytes / 2, &tmK, g * kD + 64, y, &k_full[s]);
        }
        // Extra B columns of the tile's keys: (b_hi, b_lo, b_hi, 0, ...); with a row's
        // (g_hi, g_hi, g_lo, 0, ...) the MMA adds g_hi b_hi + g_hi b_lo + g_lo b_hi, i.e.
        // g * b to ~2^-16 relative
        {
          unsigned char* bx = smem + AttnSmem::BEX + s * kExBytes;
#pragma unroll
          for (int e = 0; e < 4; ++e) attn_put_key_bias(bx, lane * 4 + e, bv[e]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bx_full[s]);
        }
        // V of tile j once both heads' PV MMAs of tile j - kStages are done
        if (!warp_all(mbar_wait(&v_empty[s], ph ^ 1u, abort_flag, p.status))) {
          ++loaded;
          break;
        }
        unsigned char* vt = smem + AttnSmem::V + s * kTileBytes;
        if (lane == 0) {
          mbar_arrive_expect_tx(&v_full[s], kTileBytes);
          tma_load_2d(vt, &tmV, g * kD, y, &v_full[s]);
          tma_load_2d(vt + kTileBytes / 2, &tmV, g * kD + 64, y, &v_full[s]);
        }
        load_bias(j + 1, bv);
        ++loaded;
        ++loaded_v;
      }
      if (lane == 0) {
        // drain: no bulk copy may still be landing when the CTA exits
        if (q_issued) mbar_wait(q_full, 0, nullptr, p.status);
        for (int j = loaded - kStages < 0 ? 0 : loaded - kStages; j < loaded; ++j) {
          const uint32_t ph = (uint32_t)(j / kStages) & 1u;
          mbar_wait(&k_full[j % kStages], ph, nullptr, p.status);
          if (j < loaded_v) mbar_wait(&v_full[j % kStages], ph, nullptr, p.status);
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      if (lane == 0) {
        constexpr uint32_t idesc_s = idesc_bf16_f32(128, kBN, false, false);
        constexpr uint32_t idesc_o = idesc_bf16_f32(128, kD, false, true);
        // Descriptors are built once; stepping along K only moves the start-address
        // field (bits 0-13, address >> 4), which cannot carry for shared addresses
        // below 256 KB.
        const uint64_t q_desc[2] = {sw128_desc(smem_u32(smem + AttnSmem::Q0), 16, 1024),
                                    sw128_desc(smem_u32(smem + AttnSmem::Q1), 16, 1024)};
        const uint64_t k_desc0 = sw128_desc(smem_u32(smem + AttnSmem::K), 16, 1024);
        const uint64_t v_desc0 = sw128_desc(smem_u32(smem + AttnSmem::V), kTileBytes / 2, 1024);
        // extra K columns (gate bias): core matrices 128 bytes apart along K, 8-row groups
        // 256 bytes apart
        const uint64_t ax_desc[2] = {
            interleave_desc(smem_u32(smem + AttnSmem::AEX), 128, 256),
            interleave_desc(smem_u32(smem + AttnSmem::AEX + kExBytes), 128, 256)};
        const uint64_t bx_desc0 = interleave_desc(smem_u32(smem + AttnSmem::BEX), 128, 256);
        const uint32_t s_col[2] = {0u, 128u};
        const uint32_t o_col[2] = {256u, 384u};
        auto issue_s = [&](int hh, int j) {
          const uint64_t kd = k_desc0 + (uint64_t)(((j % kStages) * kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t off = (uint64_t)(((kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32) >> 4);
            mma_ss(tmem + s_col[hh], q_desc[hh] + off, kd + off, idesc_s, kk != 0);
          }
          // + (gamma_h * log2(e) / t_r) * bias_c, one more K=16 step on the extra columns
          mma_ss(tmem + s_col[hh], ax_desc[hh],
                 bx_desc0 + (uint64_t)(((j % kStages) * kExBytes) >> 4), idesc_s, 1u);
          mma_commit(&s_full[hh]);
        };
        // O += P V over the tile's keys [64 half, 64 half + 64): the first half as soon
        // as the softmax has stored its P, while it computes the second
        auto issue_pv = [&](int hh, int j, int half) {
          const uint64_t vd = v_desc0 + (uint64_t)(((j % kStages) * kTileBytes) >> 4);
#pragma unroll
          for (int q = 0; q < kBN / 32; ++q) {
            const int kk = half * (kBN / 32) + q;
            // A = P (bf16 pairs in TMEM, 8 columns per 16 keys); B = V rows kk*16.. (MN-major)
            mma_ts(tmem + o_col[hh], tmem + s_col[hh] + kk * 8, vd + (uint64_t)((kk * 16 * 128) >> 4),
                   idesc_o, (j | kk) != 0);
          }
          if (half) mma_commit(&pv_done[hh]);
        };
        bool ok = mbar_wait(q_full, 0, abort_flag, p.status) &&
                  mbar_wait(&ax_ready[0], 0, abort_flag, p.status) &&
                  mbar_wait(&ax_ready[1], 0, abort_flag, p.status) &&
                  mbar_wait(&k_full[0], 0, abort_flag, p.status) &&
                  mbar_wait(&bx_full[0], 0, abort_flag, p.status);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          mma_commit(&k_empty[0]);
          for (int j = 0; j < nt && ok; ++j) {
            const int s = j % kStages;
            const uint32_t ph = (uint32_t)(j / kStages) & 1u;
            const uint32_t pj = (uint32_t)j & 1u;
            ok = mbar_wait(&v_full[s], ph, abort_flag, p.status) &&
                 mbar_wait(&p_half[0], pj, abort_flag, p.status);
            if (!ok) break;
            tc_fence_after();
            issue_pv(0, j, 0);
            if (!(ok = mbar_wait(&p_full[0], pj, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(0, j, 1);
            const bool more = j + 1 < nt;
            if (more) {
              const int s2 = (j + 1) % kStages;
              const uint32_t ph2 = (uint32_t)((j + 1) / kStages) & 1u;
              if (!(ok = mbar_wait(&k_full[s2], ph2, abort_flag, p.status) &&
                         mbar_wait(&bx_full[s2], ph2, abort_flag, p.status)))
                break;
              tc_fence_after();
              issue_s(0, j + 1);
            }
            if (!(ok = mbar_wait(&p_half[1], pj, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(1, j, 0);
            if (!(ok = mbar_wait(&p_full[1], pj, abort_flag, p.status))) break;
            tc_fence_after();
            issue_pv(1, j, 1);
            mma_commit(&v_empty[s]);
            if (more) {
              issue_s(1, j + 1);
              mma_commit(&k_empty[(j + 1) % kStages]);
            }
          }
        }
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, p.status);  // every MMA retired before TMEM is freed
      }
    }
  } else {
    regs_inc<kRegsHigh>();
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 4) >> 2;  // 0: head h0, 1: head h0 + 1
    const int hh = h0 + wg;
    const int q = warp & 3;
    const int rit = q * 32 + lane;   // row in tile
    const int r = q0 + rit;          // rank inside the request
    const bool row_valid = r < n_b;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_t = tmem + lane_off + (wg ? 128u : 0u);
    const uint32_t o_t = tmem + lane_off + (wg ? 384u : 256u);

    const double tau = attn_tau(p.beta, r, row_valid ? p.kept_pos[row0 + r] : 0);

    // The logit in the log2 domain is t * S with t = tau_r * log2(e) / sqrt(d) and
    // S = q.k + (gamma_h * log2(e) / t) * bias_c: the tensor core adds the bias term
    // through one extra K=16 step whose A columns, per row, hold g = gamma_h log2(e) / t
    // split into bf16 parts (g_hi, g_hi, g_lo).  t >= 0 (beta >= 0); t = 0 (first kept
    // token of a request whose position is not 0) is taken as 2^-66, which leaves
    // t * S = gamma_h log2(e) bias_c.
    const float t2 = attn_logit_scale(tau, kD);
    {
      attn_put_query_gain(smem + AttnSmem::AEX + wg * kExBytes, rit, p.gamma[hh] * kLog2e / t2);
      fence_proxy_async_smem();  // read by the tensor core
      mbar_arrive(&ax_ready[wg]);
    }

    float m_run = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!(ok = warp_all(mbar_wait(&s_full[wg], (uint32_t)j & 1u, abort_flag, p.status)))) break;
      tc_fence_after();
      uint32_t sv[kBN];
      tmem_ld32(s_t + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(s_t + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld32(s_t + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
      tmem_ld32(s_t + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      tmem_wait_ld();
      const float mx = t2 * ((j0 + j == qt) ? row_max<true>(sv, rit) : row_max<false>(sv, rit));
      // Lazy rescale: move the running max only when it grows by more than 2^8.
      float alpha = 1.0f;
      bool rescale = false;
      if (j == 0) {
        m_run = mx;
      } else if (mx > m_run + kRescaleThreshold) {
        alpha = ex2_approx(m_run - mx);
        m_run = mx;
        rescale = true;
      }
      // O rescale, warp-uniform (tcgen05.ld/st are warp-collective; alpha = 1 on rows
      // that keep their max), before any of this tile's P is released to the PV MMAs.
      // PV(j-1) has retired: S(j) was committed after it.
      if (__any_sync(0xFFFFFFFFu, rescale)) {
        if (!(ok = warp_all(mbar_wait(&pv_done[wg], (uint32_t)(j - 1) & 1u, abort_flag,
                                      p.status))))
          break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t ro[32];
          tmem_ld32(o_t + c * 32, ro);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = __float_as_uint(__uint_as_float(ro[i]) * alpha);
          tmem_st32(o_t + c * 32, ro);
        }
      }
      const uint64_t negm = f2pack(-m_run, -m_run);
      const uint64_t t2p = f2pack(t2, t2);
      uint64_t acc0 = f2pack(0.f, 0.f), acc1 = acc0;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int e = 64 * hf + 2 * i;
          const uint64_t d = fma2(f2pack(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])), t2p, negm);
          float x0, x1;
          f2unpack(d, x0, x1);
          const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
          if (i & 1) acc1 = add2(acc1, f2pack(p0, p1));
          else acc0 = add2(acc0, f2pack(p0, p1));
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_t + 32 * hf, pk);
        if (hf == 0) {  // keys 0..63 (and any O rescale) are in TMEM: their PV may start
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(&p_half[wg]);
        }
      }
      float a0, a1, a2, a3;
      f2unpack(acc0, a0, a1);
      f2unpack(acc1, a2, a3);
      l_sum = l_sum * alpha + ((a0 + a1) + (a2 + a3));
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
    }
    const bool done =
        ok && warp_all(mbar_wait(&pv_done[wg], (uint32_t)(nt - 1) & 1u, abort_flag, p.status));
    if (done) tc_fence_after();
    // Both heads meet here once: after it every MMA has retired, so the Q/K/V/bias
    // shared memory is free for staging, whatever path follows (all CTA-uniform).
    const bool all_done = named_bar_and(1, 256, done);
    const bool elected = warp == 4 && lane == 0;
    // A full query tile lies inside its request: its bf16 output goes through shared
    // memory (128-byte swizzle, two 64-column boxes per head) and TMA stores.  A
    // request's ragged last tile stores rows directly (a full box would reach into the
    // next request's rows).
    const bool full_tile = q0 + kBM <= n_b;
    unsigned char* out_head = smem + kEpiOut + wg * 2 * kBoxBytes;
    auto put_chunk = [&](int c, const float (&acc)[32], float inv) {
      uint32_t w[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
      if (full_tile) {
        unsigned char* box = out_head + (c >> 1) * kBoxBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = (c & 1) * 4 + u;  // 16-byte chunk of the row inside its box
          *reinterpret_cast<uint4*>(box + rit * 128 + ((k ^ (rit & 7)) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      } else if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(p.o + (row0 + r) * p.ld_o + (int64_t)hh * kD + c * 32);
#pragma unroll
        for (int u = 0; u < 4; ++u) dst[u] = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      }
    };
    auto store_lse = [&](float M, float L) {
      if (row_valid && p.lse)
        p.lse[(int64_t)hh * p.k_total + row0 + r] = (M + log2f(L)) * 0.69314718055994531f;
    };
    // after every thread has put its chunks: the staged tile goes out by TMA
    auto flush_out = [&]() {
      fence_proxy_async_smem();
      named_bar_sync(1, 256);
      if (full_tile && elected) {
        for (int h = 0; h < 2; ++h)
          for (int bx = 0; bx < 2; ++bx)
            tma_store_2d(&tmO, (h0 + h) * kD + 64 * bx, (int32_t)(row0 + q0),
                         smem + kEpiOut + (h * 2 + bx) * kBoxBytes);
        bulk_commit_group();
      }
    };
    auto own_chunk = [&](int c, float (&x)[32]) {
      uint32_t ro[32];
      tmem_ld32(o_t + c * 32, ro);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(ro[e]);
    };

    if (nparts == 1) {
      if (all_done) {
        const float inv = 1.0f / l_sum;
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          float acc[32];
          own_chunk(c, acc);
          put_chunk(c, acc, inv);
        }
        store_lse(m_run, l_sum);
        flush_out();
      }
    } else if (all_done) {
      // Split query tile.  Each part counts its arrival; every part but the last to
      // arrive publishes its partial result (unnormalised O, row max, row sum) with bulk
      // stores and raises its ready flag; the last one merges all parts, summing in part
      // order whichever part it is (so every run rounds alike):
      //   M = max_i m_i, L = sum_i 2^(m_i - M) l_i, o = sum_i 2^(m_i - M) O_i / L.
      // It waits only for parts that have already arrived and are just storing, so the
      // wait always ends.
      int* cnt = p.part_count + (int64_t)(item - part) * hg + head_grp;
      if (elected) {
        const int before = atomicAdd(cnt, 1);
        if (before < 0 || before >= nparts) {
          // the counter did not start at zero: the workspace was not zero-filled
          if (p.status) atomicOr(p.status, TG_STATUS_WORKSPACE);
          *last_part = 2;  // neither publish nor merge
        } else {
          *last_part = before == nparts - 1 ? 1 : 0;
        }
      }
      named_bar_sync(1, 256);
      float* blk_smem = reinterpret_cast<float*>(smem) + wg * kPartFloats;  // this head's block
      auto blk = [&](int i, int h) {
        return p.part_ws + ((int64_t)(item - part + i) * p.n_q_heads + h) * kPartFloats;
      };
      if (*last_part == 2) {
        // corrupt workspace: nothing to do (status set above)
      } else if (!*last_part) {
        // straight from TMEM to this head's block, one row per thread (a warp's stores
        // of one 4-column group are 512 contiguous bytes)
        float* dst = blk(part, hh);
        float4* ocol = reinterpret_cast<float4*>(dst) + rit;
#pragma unroll 1
        for (int c = 0; c < kD / 32; ++c) {
          float x[32];
          own_chunk(c, x);
#pragma unroll
          for (int u = 0; u < 8; ++u)
            __stcg(ocol + (c * 8 + u) * kBM,
                   make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]));
        }
        __stcg(dst + kBM * kD + rit, m_run);
        __stcg(dst + kBM * kD + kBM + rit, l_sum);
        __threadfence();  // this thread's rows are visible GPU-wide before the flag
        named_bar_sync(1, 256);
        if (elected) {
          fence_proxy_async_global();  // the merging part reads the block by bulk copies
          st_release_gpu(p.part_ready + (int64_t)item * hg + head_grp, 1);
        }
      } else {
        if (elected) {
          bool ready = true;
          for (int i = 0; i < nparts && ready; ++i)
            if (i != part)
              ready = wait_flag_gpu(p.part_ready + (int64_t)(item - part + i) * hg + head_grp,
                                    abort_flag, p.status);
          fence_proxy_async_global();  // the partials are read by bulk copies next
          *parts_ready = ready ? 1 : 0;
        }
        named_bar_sync(1, 256);
        const int np = nparts;
        int copies = 0;
        // stage part i's block (both heads) in shared memory; CTA-uniform outcome
        auto stage = [&](int i) {
          named_bar_sync(1, 256);  // nobody still reads the previous staged part
          if (elected) {
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(merge_full, 2 * kPartFloats * 4);
            bulk_load(smem, blk(i, h0), kPartFloats * 4, merge_full);
            bulk_load(smem + kPartFloats * 4, blk(i, h0 + 1), kPartFloats * 4, merge_full);
          }
          const bool got = named_bar_and(
              1, 256, mbar_wait(merge_full, (uint32_t)copies & 1u, abort_flag, p.status));
          ++copies;
          return got;
        };
        bool ok_m = *parts_ready != 0;
        if (ok_m && np == 2) {
          // one other part: stage it, then a single pass
          const int other = 1 - part;
          ok_m = stage(other);
          if (ok_m) {
            const float m_o = blk_smem[kBM * kD + rit], l_o = blk_smem[kBM * kD + kBM + rit];
            const float M = fmaxf(m_run, m_o);
            const float w_own = ex2_approx(m_run - M), w_o = ex2_approx(m_o - M);
            const float w0 = part == 0 ? w_own : w_o, w1 = part == 0 ? w_o : w_own;
            const float L = fmaf(w1, part == 0 ? l_o : l_sum, w0 * (part == 0 ? l_sum : l_o));
            const float inv = 1.0f / L;
            const float4* g = reinterpret_cast<const float4*>(blk_smem) + rit;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
              float own[32], acc[32];
              own_chunk(c, own);
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float4 x = g[(c * 8 + u) * kBM];
                const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float a0 = part == 0 ? own[4 * u + e] : xs[e];
                  const float a1 = part == 0 ? xs[e] : own[4 * u + e];
                  acc[4 * u + e] = fmaf(w1, a1, w0 * a0);
                }
              }
              put_chunk(c, acc, inv);
            }
            store_lse(M, L);
          }
        } else if (ok_m) {
          // several other parts: batch-load every row max and sum, then one pass per
          // part in part order with the running sum kept in the TMEM columns S used
          float mi[kMaxParts], li[kMaxParts];
#pragma unroll
          for (int i = 0; i < kMaxParts; ++i) {
            if (i < np) {
              mi[i] = i == part ? m_run : __ldcg(blk(i, hh) + kBM * kD + rit);
              li[i] = i == part ? l_sum : __ldcg(blk(i, hh) + kBM * kD + kBM + rit);
            }
          }
          float M = -INFINITY;
#pragma unroll
          for (int i = 0; i < kMaxParts; ++i)
            if (i < np) M = fmaxf(M, mi[i]);
          float L = 0.f;
#pragma unroll
          for (int i = 0; i < kMaxParts; ++i) {
            if (i < np) {
              mi[i] = ex2_approx(mi[i] - M);  // from here on: the part's weight
              L = i == 0 ? mi[i] * li[i] : fmaf(mi[i], li[i], L);
            }
          }
          const float inv = 1.0f / L;
#pragma unroll 1
          for (int i = 0; i < np && ok_m; ++i) {
            float w = mi[0];
#pragma unroll
            for (int t = 1; t < kMaxParts; ++t)
              if (t == i) w = mi[t];
            if (i != part && !(ok_m = stage(i))) break;
            const float4* g = reinterpret_cast<const float4*>(blk_smem) + rit;
#pragma unroll 1
            for (int c = 0; c < kD / 32; ++c) {
              float acc[32];
              if (i > 0) {
                uint32_t ra[32];
                tmem_ld32(s_t + c * 32, ra);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) acc[e] = __uint_as_float(ra[e]);
              }
              float x[32];
              if (i == part) {
                own_chunk(c, x);
              } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                  const float4 v4 = g[(c * 8 + u) * kBM];
                  x[4 * u] = v4.x;
                  x[4 * u + 1] = v4.y;
                  x[4 * u + 2] = v4.z;
                  x[4 * u + 3] = v4.w;
                }
              }
#pragma unroll
              for (int e = 0; e < 32; ++e) acc[e] = i == 0 ? w * x[e] : fmaf(w, x[e], acc[e]);
              if (i == np - 1) {
                put_chunk(c, acc, inv);
              } else {
                uint32_t wa[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) wa[e] = __float_as_uint(acc[e]);
                tmem_st32(s_t + c * 32, wa);
                tmem_wait_st();
              }
            }
          }
          if (ok_m) store_lse(M, L);
        }
        // after an abort: the last staged copy may still be landing in shared memory
        if (!ok_m && copies > 0 && elected)
          mbar_wait(merge_full, (uint32_t)(copies - 1) & 1u, nullptr, p.status);
        const int ok_all = named_bar_and(1, 256, ok_m);
        if (ok_all) flush_out();
        named_bar_sync(1, 256);  // every read of the partials is done
        if (elected) {  // leave the counters zeroed for the next call
          for (int i = 0; i < nparts; ++i)
            p.part_ready[(int64_t)(item - part + i) * hg + head_grp] = 0;
          *cnt = 0;
        }
      }
    }
    // TMA/bulk stores have read shared memory before the CTA exits (their global writes
    // are complete, like every other write of the grid, when the kernel is)
    if (elected) bulk_wait_read_all();
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Work plan: the key-tile chunk per item and the item count per request, chosen to
// minimise the estimated makespan over the SMs (one CTA per SM at a time).
struct AttnPlan {
  int chunk;
  int n_items;
  bool split;
};

// Makespan (in key-tile units) of launching the items of `chunk` in launch order on
// `sms` SMs, one CTA per SM at a time: the block scheduler hands each CTA to the first
// SM that frees up, which is list scheduling in launch order (heaviest first within a
// request).  Costs, measured with a global-timer trace of every CTA on a B200 (one key
// tile of both heads ~2.2 us): every CTA pays kCtaOverhead for its prologue (first MMA
// ~4.5 us after the start) and output; a part of a split tile that publishes its partial
// pays kPublish; the part that arrives last waits for the others' partials and pays
// kMergePart per other part before the tile is done.
constexpr double kCtaOverhead = 3.0;
constexpr double kPublish = 1.0;
constexpr double kMergePart = 1.3;
double simulate_makespan(const int32_t* cu_kept_host, int batch, int head_groups, int sms,
                         int chunk) {
  std::vector<double> busy((size_t)sms, 0.0);  // finish time of each SM's last CTA
  auto first_free = [&]() {
    return (int)(std::min_element(busy.begin(), busy.end()) - busy.begin());
  };
  std::vector<double> fin;
  std::vector<int> sm_of;
  for (int b = 0; b < batch; ++b) {
    const int nt = ceil_div(cu_kept_host[b + 1] - cu_kept_host[b], kBM);
    for (int qt = nt - 1; qt >= 0; --qt) {
      const int np = ceil_div(qt + 1, chunk);
      fin.assign((size_t)np * head_groups, 0.0);
      sm_of.assign((size_t)np * head_groups, 0);
      for (int part = 0; part < np; ++part) {
        const int units = std::min(qt + 1, (part + 1) * chunk) - part * chunk;
        for (int h = 0; h < head_groups; ++h) {
          const int s = first_free();
          busy[s] += units + kCtaOverhead + (np > 1 ? kPublish : 0.0);
          fin[(size_t)part * head_groups + h] = busy[s];
          sm_of[(size_t)part * head_groups + h] = s;
        }
      }
      if (np > 1) {
        for (int h = 0; h < head_groups; ++h) {
          int last = 0;
          for (int part = 1; part < np; ++part)
            if (fin[(size_t)part * head_groups + h] > fin[(size_t)last * head_groups + h])
              last = part;
          busy[sm_of[(size_t)last * head_groups + h]] =
              fin[(size_t)last * head_groups + h] + kMergePart * (np - 1);
        }
      }
    }
  }
  return *std::max_element(busy.begin(), busy.end());
}

int make_plan(const int32_t* cu_kept_host, int batch, int head_groups, int sms, AttnPlan& plan,
              int32_t* item_prefix) {
  int max_tiles = 0;
  int64_t units = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_kept_host[b + 1] - cu_kept_host[b];
    if (n < 0) return TG_ERR_INVALID_ARGUMENT;
    const int nt = ceil_div((int)n, kBM);
    max_tiles = std::max(max_tiles, nt);
    units += (int64_t)nt * (nt + 1) / 2;
  }
  // Plans are cached per layout: the gated layers of a step share one.
  static thread_local std::vector<int32_t> cached_layout;
  static thread_local AttnPlan cached_plan;
  static thread_local int cached_hg = -1, cached_sms = -1;
  std::vector<int32_t> layout(cu_kept_host, cu_kept_host + batch + 1);
  if (layout == cached_layout && cached_hg == head_groups && cached_sms == sms) {
    plan = cached_plan;
  } else {
    // Candidates: no split, and every chunk up to three times the balanced share of one
    // SM; a split must shorten the estimate by a fiftieth.
    const double share = (double)units * head_groups / sms;
    int best = std::max(max_tiles, 1);
    double best_cost = 0.98 * simulate_makespan(cu_kept_host, batch, head_groups, sms, best);
    const int c_hi = std::min(max_tiles - 1, (int)std::ceil(3.0 * share));
    for (int c = 2; c <= c_hi; ++c) {
      if (ceil_div(max_tiles, c) > kMaxParts) continue;
      const double cost = simulate_makespan(cu_kept_host, batch, head_groups, sms, c);
      if (cost < best_cost) {
        best_cost = cost;
        best = c;
      }
    }
    plan.split = best < max_tiles;
    plan.chunk = best;
    cached_layout = layout;
    cached_plan = plan;
    cached_hg = head_groups;
    cached_sms = sms;
  }
  int64_t items = 0;
  item_prefix[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int nt = ceil_div(cu_kept_host[b + 1] - cu_kept_host[b], kBM);
    for (int qt = 0; qt < nt; ++qt) items += ceil_div(qt + 1, plan.chunk);
    if (items > 0x3FFFFFFF) return TG_ERR_UNSUPPORTED_SHAPE;
    item_prefix[b + 1] = (int32_t)items;
  }
  plan.n_items = (int)items;
  return TG_OK;
}

// Split workspace: the parts' partial results, then at a 256-byte boundary two int32
// arrays indexed by (work item, head group): arrival counters (used at a tile's first
// item) and ready flags.
size_t part_bytes(int64_t n_items, int n_q_heads) {
  return ((size_t)n_items * n_q_heads * kPartFloats * sizeof(float) + 255) & ~size_t(255);
}
size_t split_workspace_bytes(int64_t n_items, int n_q_heads, int head_groups) {
  return part_bytes(n_items, n_q_heads) + 2 * (size_t)n_items * head_groups * sizeof(int32_t);
}

// The register split above assumes the kernel is launched with kLaunchRegs registers
// per thread; a smaller launch allocation would leave setmaxnreg.inc waiting forever.
int check_register_budget() {
  static int checked_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (checked_dev == dev) return TG_OK;
  cudaFuncAttributes fa;
  TG_CUDA_TRY(cudaFuncGetAttributes(&fa, gated_attention_kernel));
  if (fa.numRegs * kThreads < 128 * kRegsLow + 256 * kRegsHigh ||
      fa.maxThreadsPerBlock < kThreads)
    return TG_ERR_UNSUPPORTED_SHAPE;
  TG_CUDA_TRY(cudaFuncSetAttribute(gated_attention_kernel,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, AttnSmem::BYTES));
  checked_dev = dev;
  return TG_OK;
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" size_t tg_gated_attention_workspace_size(const int32_t* cu_kept_host, int batch,
                                                    int n_q_heads, int n_kv_heads, int head_dim) {
  if (head_dim != kD || batch <= 0 || batch > kMaxBatch || !cu_kept_host || n_kv_heads <= 0 ||
      n_q_heads <= 0 || n_q_heads % n_kv_heads || (n_q_heads / n_kv_heads) % 2)
    return 0;
  AttnPlan plan;
  static thread_local int32_t prefix[kMaxBatch + 1];
  if (make_plan(cu_kept_host, batch, n_q_heads / 2, sm_count(), plan, prefix) != TG_OK ||
      !plan.split)
    return 0;
  return split_workspace_bytes(plan.n_items, n_q_heads, n_q_heads / 2);
}

extern "C" int tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                  const tg_bf16* v, int64_t ld_v, const int32_t* cu_kept,
                                  const int32_t* cu_kept_host, int batch, int n_q_heads,
                                  int n_kv_heads, int head_dim, const int32_t* kept_pos,
                                  const float* kept_bias, const float* gamma, float beta,
                                  tg_bf16* o, int64_t ld_o, float* lse, void* workspace,
                                  size_t workspace_bytes, uint32_t* status, tg_stream_t stream) {
  if (head_dim != kD) return TG_ERR_UNSUPPORTED_SHAPE;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads) return TG_ERR_INVALID_ARGUMENT;
  const int group = n_q_heads / n_kv_heads;
  if (group % 2) return TG_ERR_UNSUPPORTED_SHAPE;
  if (batch > kMaxBatch) return TG_ERR_UNSUPPORTED_SHAPE;
  if (batch < 0 || !cu_kept_host) return TG_ERR_INVALID_ARGUMENT;
  if (batch == 0) return TG_OK;
  if (cu_kept_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  for (int b = 0; b < batch; ++b)
    if (cu_kept_host[b + 1] < cu_kept_host[b]) return TG_ERR_INVALID_ARGUMENT;
  const int64_t k_total = cu_kept_host[batch];
  if (k_total == 0) return TG_OK;
  if (!q || !k || !v || !o || !cu_kept || !kept_pos || !kept_bias || !gamma)
    return TG_ERR_INVALID_ARGUMENT;
  if (ld_q < (int64_t)n_q_heads * kD || ld_o < (int64_t)n_q_heads * kD ||
      ld_k < (int64_t)n_kv_heads * kD || ld_v < (int64_t)n_kv_heads * kD)
    return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !stride_ok(ld_q, 2) ||
      !stride_ok(ld_k, 2) || !stride_ok(ld_v, 2) || !stride_ok(ld_o, 2))
    return TG_ERR_MISALIGNED;
  if (workspace && !aligned16(workspace)) return TG_ERR_MISALIGNED;
  if (!std::isfinite(beta) || beta < 0.f) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  TG_TRY(check_register_budget());

  AttnParams prm{};
  const int head_groups = n_kv_heads * (group / 2);
  AttnPlan plan;
  TG_TRY(make_plan(cu_kept_host, batch, head_groups, sm_count(), plan, prm.item_prefix));
  const size_t need = split_workspace_bytes(plan.n_items, n_q_heads, head_groups);
  if (plan.split && (!workspace || workspace_bytes < need)) {
    // no room for partial results: one item per query tile
    int max_tiles = 1;
    for (int b = 0; b < batch; ++b)
      max_tiles = std::max(max_tiles, ceil_div(cu_kept_host[b + 1] - cu_kept_host[b], kBM));
    plan.split = false;
    plan.chunk = max_tiles;
    int items = 0;
    for (int b = 0; b < batch; ++b) {
      items += ceil_div(cu_kept_host[b + 1] - cu_kept_host[b], kBM);
      prm.item_prefix[b + 1] = items;
    }
    plan.n_items = items;
  }

  CUtensorMap tq, tk, tv, to;
  TG_TRY(make_tmap_bf16_2d(&tq, q, (uint64_t)k_total, (uint64_t)n_q_heads * kD, (uint64_t)ld_q, 64, kBM));
  TG_TRY(make_tmap_bf16_2d(&tk, k, (uint64_t)k_total, (uint64_t)n_kv_heads * kD, (uint64_t)ld_k, 64, kBN));
  TG_TRY(make_tmap_bf16_2d(&tv, v, (uint64_t)k_total, (uint64_t)n_kv_heads * kD, (uint64_t)ld_v, 64, kBN));
  TG_TRY(make_tmap_bf16_2d(&to, o, (uint64_t)k_total, (uint64_t)n_q_heads * kD, (uint64_t)ld_o, 64, kBM));
  prm.cu_kept = cu_kept;
  prm.kept_pos = kept_pos;
  prm.kept_bias = kept_bias;
  prm.gamma = gamma;
  prm.beta = beta;
  prm.o = reinterpret_cast<uint16_t*>(o);
  prm.ld_o = ld_o;
  prm.lse = lse;
  prm.k_total = k_total;
  prm.n_q_heads = n_q_heads;
  prm.group = group;
  prm.head_pairs = group / 2;
  prm.n_kv_heads = n_kv_heads;
  prm.batch = batch;
  prm.status = status;
  prm.chunk = plan.chunk;
  prm.part_ws = plan.split ? static_cast<float*>(workspace) : nullptr;
  prm.part_count = plan.split ? reinterpret_cast<int*>(static_cast<unsigned char*>(workspace) +
                                                       part_bytes(plan.n_items, n_q_heads))
                              : nullptr;
  prm.part_ready = plan.split ? prm.part_count + (int64_t)plan.n_items * head_groups : nullptr;

  const int64_t grid = (int64_t)plan.n_items * head_groups;
  if (grid > 0x7FFFFFFF) return TG_ERR_UNSUPPORTED_SHAPE;
  TG_TRY(launch(gated_attention_kernel, dim3((unsigned)grid), dim3(kThreads), AttnSmem::BYTES,
                (cudaStream_t)stream, tq, tk, tv, to, prm));
  return TG_OK;
}
