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
// One CTA = one request, one tile of 128 query ranks, one kv head and the two q
// heads (h0, h0 + 1) that read it.  Tensor memory (512 columns):
//   S0/P0 [0,128)  S1/P1 [128,256)  O0 [256,384)  O1 [384,512)
// Warps: 0 TMA producer (Q once, then K/V tiles + key bias through a 2-stage ring);
// 1 MMA issuer (S = Q K^T from shared memory, O += P V with P read from TMEM);
// 2-5 softmax of head h0, 6-9 softmax of head h1, one thread per query row (warp w
// reads TMEM lane quarter w % 4, so each group of four covers all 128 rows).  The two
// heads ping-pong: while one softmax runs, the tensor core works on the other head.
// Softmax works in the log2 domain; the running max is only moved (and O rescaled in
// TMEM) when it grows by more than 2^8, which keeps P within bf16 range.
#include <cuda.h>

#include <cmath>
#include <cstdint>

#include "tg_host.h"
#include "tg_ptx.cuh"

namespace tg {
namespace {

constexpr int kD = 128;         // head_dim
constexpr int kBM = 128;        // query rows per tile
constexpr int kBN = 128;        // keys per KV tile
constexpr int kStages = 2;      // K/V ring depth
constexpr int kThreads = 320;   // 10 warps
constexpr int kMaxBatch = 512;  // requests per call (tile table lives in the parameters)
constexpr int kTileBytes = kBM * kD * 2;  // 32 KB: 128 rows x 128 bf16, two 64-column boxes
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;

struct AttnSmem {
  // 1024-aligned tiles first
  static constexpr int Q0 = 0;
  static constexpr int Q1 = Q0 + kTileBytes;
  static constexpr int K = Q1 + kTileBytes;
  static constexpr int V = K + kStages * kTileBytes;
  static constexpr int BIAS = V + kStages * kTileBytes;
  static constexpr int BAR = BIAS + kStages * kBN * 4;
  static constexpr int END = BAR + 256;
  static constexpr int BYTES = END + 1024;  // alignment slack
};

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
  int32_t tile_prefix[kMaxBatch + 1];  // q tiles before request b
};

#ifndef TG_ATTN_MAXNREG
#define TG_ATTN_MAXNREG 168  // 320 threads: the per-block limit is taken in 128-thread units
#endif
__global__ void __maxnreg__(TG_ATTN_MAXNREG)
    gated_attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV,
                           const __grid_constant__ AttnParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* bias_s = reinterpret_cast<float*>(smem + AttnSmem::BIAS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + AttnSmem::BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;             // [kStages]
  uint64_t* v_full = k_full + kStages;     // [kStages]
  uint64_t* kv_empty = v_full + kStages;   // [kStages]
  uint64_t* s_full = kv_empty + kStages;   // [2]
  uint64_t* p_full = s_full + 2;           // [2]
  uint64_t* pv_done = p_full + 2;          // [2]
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- which tile: heads vary fastest, then q tiles heaviest-first within a request
  const int hg = p.n_kv_heads * p.head_pairs;
  const int head_grp = blockIdx.x % hg;
  const int t = blockIdx.x / hg;
  int b = 0;
  {
    int lo = 0, hi = p.batch;  // largest b with tile_prefix[b] <= t
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.tile_prefix[mid] <= t) lo = mid; else hi = mid;
    }
    b = lo;
  }
  const int ntiles_b = p.tile_prefix[b + 1] - p.tile_prefix[b];
  const int qt = ntiles_b - 1 - (t - p.tile_prefix[b]);
  const int g = head_grp / p.head_pairs;
  const int h0 = g * p.group + 2 * (head_grp % p.head_pairs);
  const int64_t row0 = p.cu_kept[b];
  const int n_b = p.cu_kept[b + 1] - p.cu_kept[b];
  const int q0 = qt * kBM;
  const int nt = qt + 1;  // causal: key tiles 0..qt

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 2);  // TMA bytes + key-bias stores
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&s_full[h], 1);
      mbar_init(&p_full[h], 128);
      mbar_init(&pv_done[h], 1);
    }
    mbar_init(drain, 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int loaded = 0;
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
    for (int j = 0; j < nt; ++j) {
      const int s = j % kStages;
      const uint32_t ph = (uint32_t)(j / kStages) & 1u;
      if (!warp_all(mbar_wait(&kv_empty[s], ph ^ 1u, abort_flag, p.status))) break;
      const int k0 = j * kBN;
      const int y = (int)(row0 + k0);
      unsigned char* kt = smem + AttnSmem::K + s * kTileBytes;
      unsigned char* vt = smem + AttnSmem::V + s * kTileBytes;
      if (lane == 0) {
        mbar_arrive_expect_tx(&k_full[s], kTileBytes);
        tma_load_2d(kt, &tmK, g * kD, y, &k_full[s]);
        tma_load_2d(kt + kTileBytes / 2, &tmK, g * kD + 64, y, &k_full[s]);
        mbar_arrive_expect_tx(&v_full[s], kTileBytes);
        tma_load_2d(vt, &tmV, g * kD, y, &v_full[s]);
        tma_load_2d(vt + kTileBytes / 2, &tmV, g * kD + 64, y, &v_full[s]);
      }
      float* bsl = bias_s + s * kBN;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int c = k0 + lane * 4 + e;
        bsl[lane * 4 + e] = c < n_b ? p.kept_bias[row0 + c] : 0.0f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&k_full[s]);
      ++loaded;
    }
    if (lane == 0) {
      // drain: no bulk copy may still be landing when the CTA exits
      if (q_issued) mbar_wait(q_full, 0, nullptr, p.status);
      for (int j = loaded - kStages < 0 ? 0 : loaded - kStages; j < loaded; ++j) {
        const uint32_t ph = (uint32_t)(j / kStages) & 1u;
        mbar_wait(&k_full[j % kStages], ph, nullptr, p.status);
        mbar_wait(&v_full[j % kStages], ph, nullptr, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kBN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, kD, false, true);
      const uint32_t q_addr[2] = {smem_u32(smem + AttnSmem::Q0), smem_u32(smem + AttnSmem::Q1)};
      const uint32_t s_col[2] = {0u, 128u};
      const uint32_t o_col[2] = {256u, 384u};
      auto issue_s = [&](int hh, int j) {
        const uint32_t k_addr = smem_u32(smem + AttnSmem::K + (j % kStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kTileBytes / 2) + (kk & 3) * 32;
          mma_ss(tmem + s_col[hh], sw128_desc(q_addr[hh] + off, 16, 1024),
                 sw128_desc(k_addr + off, 16, 1024), idesc_s, kk != 0);
        }
        mma_commit(&s_full[hh]);
      };
      auto issue_pv = [&](int hh, int j) {
        const uint32_t v_addr = smem_u32(smem + AttnSmem::V + (j % kStages) * kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          // A = P (bf16 pairs in TMEM, 8 columns per 16 keys); B = V rows kk*16.. (MN-major)
          mma_ts(tmem + o_col[hh], tmem + s_col[hh] + kk * 8,
                 sw128_desc(v_addr + kk * 16 * 128, kTileBytes / 2, 1024), idesc_o,
                 (j | kk) != 0);
        }
        mma_commit(&pv_done[hh]);
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status) &&
                mbar_wait(&k_full[0], 0, abort_flag, p.status);
      if (ok) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        for (int j = 0; j < nt && ok; ++j) {
          const int s = j % kStages;
          const uint32_t ph = (uint32_t)(j / kStages) & 1u;
          const uint32_t pj = (uint32_t)j & 1u;
          ok = mbar_wait(&v_full[s], ph, abort_flag, p.status) &&
               mbar_wait(&p_full[0], pj, abort_flag, p.status);
          if (!ok) break;
          tc_fence_after();
          issue_pv(0, j);
          const bool more = j + 1 < nt;
          if (more) {
            const int s2 = (j + 1) % kStages;
            const uint32_t ph2 = (uint32_t)((j + 1) / kStages) & 1u;
            if (!(ok = mbar_wait(&k_full[s2], ph2, abort_flag, p.status))) break;
            tc_fence_after();
            issue_s(0, j + 1);
          }
          if (!(ok = mbar_wait(&p_full[1], pj, abort_flag, p.status))) break;
          tc_fence_after();
          issue_pv(1, j);
          mma_commit(&kv_empty[s]);
          if (more) issue_s(1, j + 1);
        }
      }
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, p.status);  // every MMA retired before TMEM is freed
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int wg = (warp - 2) >> 2;  // 0: head h0, 1: head h0 + 1
    const int hh = h0 + wg;
    const int q = warp & 3;
    const int rit = q * 32 + lane;   // row in tile
    const int r = q0 + rit;          // rank inside the request
    const bool row_valid = r < n_b;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t s_t = tmem + lane_off + (wg ? 128u : 0u);
    const uint32_t o_t = tmem + lane_off + (wg ? 384u : 256u);

    double tau = (double)p.beta;
    if (row_valid) {
      const int pos = p.kept_pos[row0 + r];
      if (pos > 0) tau = (double)p.beta * log((double)r + 1.0) / log((double)pos + 1.0);
    }
    const float tau2 = (float)(tau / sqrt((double)kD) * 1.4426950408889634);
    const float gb = p.gamma[hh] * kLog2e;

    float m_run = -INFINITY, l_sum = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!(ok = warp_all(mbar_wait(&s_full[wg], (uint32_t)j & 1u, abort_flag, p.status)))) break;
      tc_fence_after();
      uint32_t sv[kBN];
      const float* bsl = bias_s + (j % kStages) * kBN;
      const bool diag = (j == qt);
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < kBN / 32; ++c) {
        // one 32-column chunk at a time keeps only 32 bias values in flight
        tmem_ld32(s_t + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * c]));
        tmem_wait_ld();
#pragma unroll
        for (int i = 32 * c; i < 32 * c + 32; ++i) {
          float v = fmaf(__uint_as_float(sv[i]), tau2, gb * bsl[i]);
          if (diag && i > rit) v = -INFINITY;
          sv[i] = __float_as_uint(v);
          mx = fmaxf(mx, v);
        }
      }
      // Lazy rescale: move the running max only when it grows by more than 2^8.
      float alpha = 1.0f;
      bool rescale = false;
      if (j == 0) {
        m_run = mx;
      } else if (mx > m_run + kRescaleThreshold) {
        alpha = exp2f(m_run - mx);
        m_run = mx;
        rescale = true;
      }
      float rs = 0.f;
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = exp2f(__uint_as_float(sv[64 * hf + 2 * i]) - m_run);
          const float p1 = exp2f(__uint_as_float(sv[64 * hf + 2 * i + 1]) - m_run);
          rs += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        tmem_st32(s_t + 32 * hf, pk);
      }
      l_sum = l_sum * alpha + rs;
      // O rescale, warp-uniform (tcgen05.ld/st are warp-collective; alpha = 1 on rows
      // that keep their max).  PV(j-1) has retired: S(j) was committed after it.
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
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&p_full[wg]);
    }
    if (ok && warp_all(mbar_wait(&pv_done[wg], (uint32_t)(nt - 1) & 1u, abort_flag, p.status))) {
      tc_fence_after();
      const float inv = 1.0f / l_sum;
      uint16_t* orow = p.o + (row0 + r) * p.ld_o + (int64_t)hh * kD;
#pragma unroll 1
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t ro[32];
        tmem_ld32(o_t + c * 32, ro);
        tmem_wait_ld();
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(ro[u * 8 + 0]) * inv, __uint_as_float(ro[u * 8 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(ro[u * 8 + 2]) * inv, __uint_as_float(ro[u * 8 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(ro[u * 8 + 4]) * inv, __uint_as_float(ro[u * 8 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(ro[u * 8 + 6]) * inv, __uint_as_float(ro[u * 8 + 7]) * inv);
            dst[u] = w;
          }
        }
      }
      if (row_valid && p.lse)
        p.lse[(int64_t)hh * p.k_total + row0 + r] = (m_run + log2f(l_sum)) * 0.69314718055994531f;
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace tg

using namespace tg;

extern "C" int tg_gated_attention(const tg_bf16* q, int64_t ld_q, const tg_bf16* k, int64_t ld_k,
                                  const tg_bf16* v, int64_t ld_v, const int32_t* cu_kept,
                                  const int32_t* cu_kept_host, int batch, int n_q_heads,
                                  int n_kv_heads, int head_dim, const int32_t* kept_pos,
                                  const float* kept_bias, const float* gamma, float beta,
                                  tg_bf16* o, int64_t ld_o, float* lse, uint32_t* status,
                                  tg_stream_t stream) {
  if (head_dim != kD) return TG_ERR_UNSUPPORTED_SHAPE;
  if (n_q_heads <= 0 || n_kv_heads <= 0 || n_q_heads % n_kv_heads) return TG_ERR_INVALID_ARGUMENT;
  const int group = n_q_heads / n_kv_heads;
  if (group % 2) return TG_ERR_UNSUPPORTED_SHAPE;
  if (batch < 0 || batch > kMaxBatch || !cu_kept_host) return batch > kMaxBatch ? TG_ERR_UNSUPPORTED_SHAPE : TG_ERR_INVALID_ARGUMENT;
  if (batch == 0) return TG_OK;
  if (cu_kept_host[0] != 0) return TG_ERR_INVALID_ARGUMENT;
  AttnParams prm{};
  int tiles = 0;
  prm.tile_prefix[0] = 0;
  for (int b = 0; b < batch; ++b) {
    const int64_t n = (int64_t)cu_kept_host[b + 1] - cu_kept_host[b];
    if (n < 0) return TG_ERR_INVALID_ARGUMENT;
    tiles += (int)((n + kBM - 1) / kBM);
    prm.tile_prefix[b + 1] = tiles;
  }
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
  if (!std::isfinite(beta)) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());

  CUtensorMap tq, tk, tv;
  TG_TRY(make_tmap_bf16_2d(&tq, q, (uint64_t)k_total, (uint64_t)n_q_heads * kD, (uint64_t)ld_q, 64, kBM));
  TG_TRY(make_tmap_bf16_2d(&tk, k, (uint64_t)k_total, (uint64_t)n_kv_heads * kD, (uint64_t)ld_k, 64, kBN));
  TG_TRY(make_tmap_bf16_2d(&tv, v, (uint64_t)k_total, (uint64_t)n_kv_heads * kD, (uint64_t)ld_v, 64, kBN));
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

  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(gated_attention_kernel,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     AttnSmem::BYTES));
    attr_dev = dev;
  }
  const int64_t grid = (int64_t)tiles * n_kv_heads * (group / 2);
  if (grid > 0x7FFFFFFF) return TG_ERR_UNSUPPORTED_SHAPE;
  gated_attention_kernel<<<(unsigned)grid, kThreads, AttnSmem::BYTES, (cudaStream_t)stream>>>(
      tq, tk, tv, prm);
  return check_launch();
}
