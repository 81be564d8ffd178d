// Dense projections of the gated layers on the kept rows (Wq/Wk/Wv with a folded
// pre-attention RMSNorm, Wo with a fused residual add), on the tcgen05 GEMM.
#include "tg_gemm.cuh"
#include "tg_host.h"

namespace tg {

template <int BN, int STAGES, int EPI>
int launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                cudaStream_t stream) {
  using Cfg = GemmCfg<BN, STAGES>;
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(gemm_kernel<BN, STAGES, EPI>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM));
    attr_dev = dev;
  }
  dim3 grid((unsigned)((p.M + Cfg::BM - 1) / Cfg::BM), (unsigned)(p.N / BN));
  gemm_kernel<BN, STAGES, EPI><<<grid, Cfg::THREADS, Cfg::SMEM, stream>>>(ta, tb, p);
  return check_launch();
}

// Explicit instantiations used by the entry points.
template int launch_gemm<256, 4, EpiStore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);
template int launch_gemm<128, 3, EpiStore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);
template int launch_gemm<256, 4, EpiScore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);

}  // namespace tg

using namespace tg;

extern "C" int tg_linear(const tg_bf16* a, int64_t lda, const tg_bf16* w, int64_t ldw, tg_bf16* c,
                         int64_t ldc, int64_t M, int N, int K, int rmsnorm_a, float eps,
                         const tg_bf16* residual, int64_t ld_res, uint32_t* status,
                         tg_stream_t stream) {
  if (M < 0 || N <= 0 || K <= 0 || (N % 128) || (K % 64)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return TG_OK;
  if (!a || !w || !c) return TG_ERR_INVALID_ARGUMENT;
  if (lda < K || ldw < K || ldc < N || (residual && ld_res < N)) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(a) || !aligned16(w) || !aligned16(c) || (residual && !aligned16(residual)) ||
      !stride_ok(lda, 2) || !stride_ok(ldw, 2) || !stride_ok(ldc, 2) ||
      (residual && !stride_ok(ld_res, 2)))
    return TG_ERR_MISALIGNED;
  if (rmsnorm_a && !(eps >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());

  // Tile width: the choice that wastes the fewest SM slots in the last wave.  BN=256
  // runs one CTA per SM, BN=128 two (smaller ring), so both fill 148 SMs per wave.
  const int64_t mt = (M + 127) / 128;
  const int sms = sm_count();
  auto eff = [&](int64_t tiles, int64_t slots) {
    const int64_t waves = (tiles + slots - 1) / slots;
    return (double)tiles / (double)(waves * slots);
  };
  const bool can256 = (N % 256) == 0;
  const double e256 = can256 ? eff(mt * (N / 256), sms) : -1.0;
  const double e128 = eff(mt * (N / 128), 2 * (int64_t)sms);
  const int bn = (can256 && e256 >= e128) ? 256 : 128;

  CUtensorMap ta, tb;
  TG_TRY(make_tmap_bf16_2d(&ta, a, (uint64_t)M, (uint64_t)K, (uint64_t)lda, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&tb, w, (uint64_t)N, (uint64_t)K, (uint64_t)ldw, 64, bn));
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = K;
  p.rmsnorm = rmsnorm_a ? 1 : 0;
  p.eps = eps;
  p.c = reinterpret_cast<uint16_t*>(c);
  p.ldc = ldc;
  p.residual = reinterpret_cast<const uint16_t*>(residual);
  p.ldr = ld_res;
  p.status = status;
  if (bn == 256) return launch_gemm<256, 4, EpiStore>(ta, tb, p, (cudaStream_t)stream);
  return launch_gemm<128, 3, EpiStore>(ta, tb, p, (cudaStream_t)stream);
}
