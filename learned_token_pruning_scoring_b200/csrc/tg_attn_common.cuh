// Arithmetic shared by the token-gated attention forward and backward kernels, so that
// the backward recomputes exactly the logits the forward normalised.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace tg {

constexpr float kAttnLog2e = 1.4426950408889634f;

// Temperature of query rank r (0-based, within its request) at original position pos:
// tau = beta * ln(r + 1) / ln(pos + 1), and tau = beta at pos = 0 (the limit r = pos).
// Evaluated in double.
__device__ __forceinline__ double attn_tau(float beta, int r, int pos) {
  double tau = (double)beta;
  if (pos > 0) tau = (double)beta * log((double)r + 1.0) / log((double)pos + 1.0);
  return tau;
}

// Scale of q.k in the log2 domain, t = tau * log2(e) / sqrt(head_dim), in fp32, floored at
// 2^-66 so that tau = 0 rows (first kept token at a non-zero position) stay finite.
__device__ __forceinline__ float attn_logit_scale(double tau, int head_dim) {
  const float t = (float)(tau / sqrt((double)head_dim) * 1.4426950408889634);
  return fmaxf(t, 0x1p-66f);
}

// x ~ hi + lo with both parts bf16 (round to nearest): hi carries 8 significant bits,
// lo the next 8.
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  const __nv_bfloat16 l = __float2bfloat16_rn(x - __bfloat162float(h));
  hi = *reinterpret_cast<const uint16_t*>(&h);
  lo = *reinterpret_cast<const uint16_t*>(&l);
}

// The gate bias enters the q.k MMA as one more K=16 step on a 128 x 16 bf16 operand pair
// in the no-swizzle core-matrix layout (8-row x 16-byte core matrices; the two along K
// 128 bytes apart, 8-row groups 256 bytes apart).  One side holds, per row,
// (b_hi, b_lo, b_hi, 0, ...) of the key bias, the other (g_hi, g_hi, g_lo, 0, ...) of the
// query's gain g = gamma * log2(e) / t, so the step adds g_hi b_hi + g_hi b_lo + g_lo b_hi,
// i.e. g * b to ~2^-16 relative.
constexpr int kAttnExBytes = 128 * 16 * 2;
__host__ __device__ constexpr int attn_ex_off(int row, int chunk) {
  return (row >> 3) * 256 + chunk * 128 + (row & 7) * 16;
}
__device__ __forceinline__ void attn_put_key_bias(unsigned char* ex, int row, float b) {
  uint16_t hi, lo;
  split_bf16(b, hi, lo);
  *reinterpret_cast<uint4*>(ex + attn_ex_off(row, 0)) =
      make_uint4((uint32_t)hi | ((uint32_t)lo << 16), hi, 0u, 0u);
  *reinterpret_cast<uint4*>(ex + attn_ex_off(row, 1)) = make_uint4(0u, 0u, 0u, 0u);
}
__device__ __forceinline__ void attn_put_query_gain(unsigned char* ex, int row, float g) {
  uint16_t hi, lo;
  split_bf16(g, hi, lo);
  *reinterpret_cast<uint4*>(ex + attn_ex_off(row, 0)) =
      make_uint4((uint32_t)hi | ((uint32_t)hi << 16), lo, 0u, 0u);
  *reinterpret_cast<uint4*>(ex + attn_ex_off(row, 1)) = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace tg
