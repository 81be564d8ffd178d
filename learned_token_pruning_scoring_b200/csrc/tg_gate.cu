// Gate scoring: fused RMSNorm + scoring MLP on tcgen05, then the sequence RMSNorm.
//
// Sources: "TokenGate 长上下文预填充提速 11.3 倍，斯坦福伯克利开源门控剪枝", section
// 门控到底插在模型的哪个位置 (a small MLP scores each token's normalised residual; the
// scores are RMSNorm-normalised along the sequence); "斯坦福与 UC Berkeley 提出 TokenGate：
// token 门控注意力让长上下文预填充最高快 11.3 倍", section "How does TokenGate learned token
// pruning work?" (the residual is the post-attention residual at the gate layer).
//
// Kernel 1 (tcgen05 GEMM, EpiScore): h[T, H] x W1[F, H]^T with F = 256 as one N tile;
//   the epilogue applies the row RMS, SiLU and the dot with w2, writes s[T] and the
//   sum of s^2 over each 32-row chunk.
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
