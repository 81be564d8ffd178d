// Dense projections of the gated layers on the kept rows (Wq/Wk/Wv with a folded
// pre-attention RMSNorm and optional QK-norm, Wo with a fused residual add, the SwiGLU
// MLP of a full layer body), on the tcgen05 GEMM, plus the one-time weight packing
// those projections read.
#include "tg_gemm.cuh"
#include "tg_host.h"

#include <algorithm>

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
  return launch(gemm_kernel<BN, STAGES, EPI>, grid, dim3(Cfg::THREADS), Cfg::SMEM, stream, ta, tb,
                p);
}

// Stream-K workspace: the partial sums of one contributing piece per cluster (two CTAs x
// two epilogue groups x 128 rows x 128 fp32 columns) and its ready flags.
size_t split_part_bytes(int clusters) { return (size_t)clusters * 4 * 32 * 128 * sizeof(float4); }
size_t split_workspace_bytes(int clusters) {
  return split_part_bytes(clusters) + (((size_t)clusters * 4 * sizeof(int) + 255) & ~size_t(255));
}

// Whether to share the last round's tiles along K (stream-K tail), and how.  The plain
// persistent launch runs ceil(tiles / C) rounds of nk k-blocks; the split one runs the
// whole rounds and then tail_units / C k-blocks per cluster plus the fixup (estimated at
// kSplitFixup k-blocks).  Split when that saves at least 7%, no tile has more than
// kMaxPieces pieces, and the caller gave a large enough workspace.
constexpr double kSplitFixup = 3.0;
PairSplit plan_split(int64_t tiles, int nk, int clusters, void* ws, size_t ws_bytes) {
  PairSplit sp{nullptr, nullptr, 0, 0};
  if (!ws || ws_bytes < split_workspace_bytes(clusters) || clusters < 2) return sp;
  const int64_t rounds = tiles / clusters;
  const int64_t tail = tiles - rounds * clusters;
  if (tail == 0) return sp;
  const int64_t tail_units = tail * nk;
  const int64_t per = tail_units / clusters;
  if (per < 1 || per * (kMaxPieces - 1) < nk) return sp;
  const double plain = (double)((tiles + clusters - 1) / clusters) * nk;
  const double split = (double)rounds * nk + (double)(tail_units + clusters - 1) / clusters +
                       kSplitFixup;
  if (split > 0.93 * plain) return sp;
  unsigned char* w = static_cast<unsigned char*>(ws);
  sp.part = reinterpret_cast<float4*>(w);
  sp.flag = reinterpret_cast<int*>(w + split_part_bytes(clusters));
  sp.dp_tiles = (int)(rounds * clusters);
  sp.tail_units = tail_units;
  return sp;
}

// The pair kernel's setmaxnreg split (PairCfg::REGS_LOW / REGS_HIGH) needs a launch
// allocation of at least PairCfg::REGS_LAUNCH_MIN registers per thread; with fewer,
// setmaxnreg.inc would wait forever, so such a build is refused before any launch.
template <typename K>
int pair_register_check(K kern, int& checked_dev) {
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (checked_dev == dev) return TG_OK;
  cudaFuncAttributes fa;
  TG_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
  if (fa.numRegs < PairCfg<1>::REGS_LAUNCH_MIN || fa.maxThreadsPerBlock < PairCfg<1>::THREADS)
    return TG_ERR_UNSUPPORTED_SHAPE;
  checked_dev = dev;
  return TG_OK;
}

template <int STAGES, int EPI>
int launch_pair(const PairMaps& maps, const GemmParams& p, cudaStream_t stream,
                void* ws = nullptr, size_t ws_bytes = 0) {
  using Cfg = PairCfg<STAGES>;
  auto kern = gemm_pair_kernel<STAGES, EPI, EPI, false>;
  auto kern_split = gemm_pair_kernel<STAGES, EPI, EPI, true>;
  static int regs_dev = -1, regs_dev_split = -1;
  TG_TRY(pair_register_check(kern, regs_dev));
  TG_TRY(pair_register_check(kern_split, regs_dev_split));
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM));
    TG_CUDA_TRY(cudaFuncSetAttribute(kern_split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     Cfg::SMEM));
    attr_dev = dev;
  }
  PairJob j0{maps, p}, j1{};
  j1.p.M = 0;  // no second job
  // persistent: at most one cluster (two CTAs) per SM pair, each walking its tiles
  const int64_t tiles = ((p.M + 255) / 256) * (p.N / Cfg::BN);
  const int all_clusters = std::max(1, sm_count() / 2);
  const PairSplit sp = plan_split(tiles, p.K / Cfg::BK, all_clusters, ws, ws_bytes);
  if (!sp.part) {
    const int64_t clusters = std::min<int64_t>(tiles, all_clusters);
    return launch(kern, dim3((unsigned)(2 * clusters)), dim3(Cfg::THREADS), Cfg::SMEM, stream,
                  j0, j1, PairChain{nullptr, nullptr, 0}, sp);
  }
  // a finishing piece waits for pieces of other clusters: all must be resident at once
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * all_clusters));
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = launch_overlap() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e =
      cudaLaunchKernelEx(&cfg, kern_split, j0, j1, PairChain{nullptr, nullptr, 0}, sp);
  if (e != cudaSuccess) {
    set_cuda_error(e);
    return TG_ERR_CUDA;
  }
  return TG_OK;
}

// Two chained jobs in one persistent launch (job 1 reads rows job 0 writes).  Every
// cluster must be resident at once, because a job-1 tile can wait for a job-0 tile of
// another cluster: the launch is cooperative, which guarantees that or fails.
template <int STAGES, int EPI0, int EPI1>
int launch_pair_chain(const PairJob& j0, const PairJob& j1, const PairChain& chain,
                      cudaStream_t stream) {
  using Cfg = PairCfg<STAGES>;
  auto kern = gemm_pair_kernel<STAGES, EPI0, EPI1, false>;
  static int regs_dev = -1;
  TG_TRY(pair_register_check(kern, regs_dev));
  static int attr_dev = -1;
  int dev = 0;
  TG_CUDA_TRY(cudaGetDevice(&dev));
  if (attr_dev != dev) {
    TG_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM));
    attr_dev = dev;
  }
  const int64_t tiles = ((j0.p.M + 255) / 256) * (j0.p.N / Cfg::BN) +
                        ((j1.p.M + 255) / 256) * (j1.p.N / Cfg::BN);
  const int64_t clusters = std::min<int64_t>(tiles, std::max(1, sm_count() / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = launch_overlap() ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  TG_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, j0, j1, chain, PairSplit{nullptr, nullptr, 0, 0}));
  return TG_OK;
}

constexpr int kPairStages = 5;

// Explicit instantiations used by the entry points.
template int launch_gemm<256, 4, EpiStore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);
template int launch_gemm<128, 3, EpiStore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);
template int launch_gemm<256, 4, EpiScore>(const CUtensorMap&, const CUtensorMap&,
                                           const GemmParams&, cudaStream_t);
template int launch_gemm<256, 4, EpiQKV>(const CUtensorMap&, const CUtensorMap&,
                                         const GemmParams&, cudaStream_t);
template int launch_gemm<128, 3, EpiQKV>(const CUtensorMap&, const CUtensorMap&,
                                         const GemmParams&, cudaStream_t);

// Tile width that wastes the fewest SM slots in the last wave: BN=256 runs one CTA
// per SM, BN=128 two (smaller ring), so both fill all SMs per wave.
int pick_bn(int64_t M, int N) {
  const int64_t mt = (M + 127) / 128;
  const int sms = sm_count();
  auto eff = [&](int64_t tiles, int64_t slots) {
    const int64_t waves = (tiles + slots - 1) / slots;
    return (double)tiles / (double)(waves * slots);
  };
  const bool can256 = (N % 256) == 0;
  const double e256 = can256 ? eff(mt * (N / 256), sms) : -1.0;
  const double e128 = eff(mt * (N / 128), 2 * (int64_t)sms);
  return (can256 && e256 >= e128) ? 256 : 128;
}

// Output projection as a pair-kernel job: c = a w^T (+ residual), row sums of squares.
int out_proj_job(PairJob& j, const tg_bf16* a, int64_t lda, const tg_bf16* w, int64_t ldw,
                 tg_bf16* c, int64_t ldc, int64_t M, int N, int K, const tg_bf16* residual,
                 int64_t ld_res, float* row_ssq_out, int64_t ld_ssq_out, uint32_t* status) {
  TG_TRY(make_tmap_bf16_2d(&j.maps.a, a, (uint64_t)M, (uint64_t)K, (uint64_t)lda, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.b, w, (uint64_t)N, (uint64_t)K, (uint64_t)ldw, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.out[0], c, (uint64_t)M, (uint64_t)N, (uint64_t)ldc, 64, 128));
  j.maps.out[1] = j.maps.out[2] = j.maps.res = j.maps.out[0];
  if (residual)
    TG_TRY(make_tmap_bf16_2d(&j.maps.res, residual, (uint64_t)M, (uint64_t)N, (uint64_t)ld_res,
                             64, 128));
  j.p = GemmParams{};
  j.p.M = M;
  j.p.N = N;
  j.p.K = K;
  j.p.c = reinterpret_cast<uint16_t*>(c);
  j.p.ldc = ldc;
  j.p.residual = reinterpret_cast<const uint16_t*>(residual);
  j.p.ldr = ld_res;
  j.p.row_ssq_out = row_ssq_out;
  j.p.ld_ssq_out = ld_ssq_out;
  j.p.status = status;
  return TG_OK;
}

// QKV projection with the folded RMSNorm (row sums of squares given), RoPE and the
// KV-cache write, as a pair-kernel job.
int qkv_job(PairJob& j, const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv, int64_t ld_w,
            int64_t M, int hidden, int q_cols, int kv_cols, float eps, const int32_t* pos,
            const float* cos_sin, int max_pos, tg_bf16* q_out, int64_t ld_q, tg_bf16* cache_k,
            tg_bf16* cache_v, int64_t ld_cache, int64_t slot_offset, const float* row_ssq_in,
            int64_t ld_ssq_in, uint32_t* status, const float* q_norm_w = nullptr,
            const float* k_norm_w = nullptr) {
  const int N = q_cols + 2 * kv_cols;
  tg_bf16* k_rows = cache_k + slot_offset * ld_cache;
  tg_bf16* v_rows = cache_v + slot_offset * ld_cache;
  TG_TRY(make_tmap_bf16_2d(&j.maps.a, x, (uint64_t)M, (uint64_t)hidden, (uint64_t)ld_x, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.b, w_qkv, (uint64_t)N, (uint64_t)hidden, (uint64_t)ld_w, 64,
                           128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.out[0], q_out, (uint64_t)M, (uint64_t)q_cols, (uint64_t)ld_q,
                           64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.out[1], k_rows, (uint64_t)M, (uint64_t)kv_cols,
                           (uint64_t)ld_cache, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.out[2], v_rows, (uint64_t)M, (uint64_t)kv_cols,
                           (uint64_t)ld_cache, 64, 128));
  j.maps.res = j.maps.out[0];
  j.p = GemmParams{};
  j.p.M = M;
  j.p.N = N;
  j.p.K = hidden;
  j.p.rmsnorm = 1;
  j.p.eps = eps;
  j.p.c = reinterpret_cast<uint16_t*>(q_out);
  j.p.ldc = ld_q;
  j.p.pos = pos;
  j.p.cos_sin = cos_sin;
  j.p.max_pos = max_pos;
  j.p.q_cols = q_cols;
  j.p.k_cols = kv_cols;
  j.p.k_out = reinterpret_cast<uint16_t*>(k_rows);
  j.p.v_out = reinterpret_cast<uint16_t*>(v_rows);
  j.p.ld_kv = ld_cache;
  j.p.row_ssq_in = row_ssq_in;
  j.p.ld_ssq_in = ld_ssq_in;
  j.p.q_norm_w = q_norm_w;
  j.p.k_norm_w = k_norm_w;
  j.p.qk_eps = eps;
  j.p.status = status;
  return TG_OK;
}

// SwiGLU up-projection as a pair-kernel job: h = SiLU(a Wg^T) * (a Wu^T), a = RMSNorm(x)
// from the row sums of squares, W rows interleaved in blocks of 64 (gate, up).
int swiglu_job(PairJob& j, const tg_bf16* x, int64_t ld_x, const tg_bf16* w_gu, int64_t ld_w,
               int64_t M, int hidden, int ffn, float eps, const float* row_ssq_in,
               int64_t ld_ssq_in, tg_bf16* h_out, int64_t ld_h, uint32_t* status) {
  TG_TRY(make_tmap_bf16_2d(&j.maps.a, x, (uint64_t)M, (uint64_t)hidden, (uint64_t)ld_x, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.b, w_gu, (uint64_t)(2 * ffn), (uint64_t)hidden, (uint64_t)ld_w,
                           64, 128));
  TG_TRY(make_tmap_bf16_2d(&j.maps.out[0], h_out, (uint64_t)M, (uint64_t)ffn, (uint64_t)ld_h, 64,
                           128));
  j.maps.out[1] = j.maps.out[2] = j.maps.res = j.maps.out[0];
  j.p = GemmParams{};
  j.p.M = M;
  j.p.N = 2 * ffn;
  j.p.K = hidden;
  j.p.rmsnorm = 1;
  j.p.eps = eps;
  j.p.c = reinterpret_cast<uint16_t*>(h_out);
  j.p.ldc = ld_h;
  j.p.row_ssq_in = row_ssq_in;
  j.p.ld_ssq_in = ld_ssq_in;
  j.p.status = status;
  return TG_OK;
}

// out[r, c] = bf16(src(r)[c] * norm_w[c]) (norm_w optional).  src(r) is row r of a, or
// with `interleave` row 64 (r / 128) + r % 64 of a (r % 128 < 64) or of b (otherwise).
__global__ void pack_rows_kernel(const uint16_t* __restrict__ a, int64_t lda,
                                 const uint16_t* __restrict__ b, int64_t ldb, int64_t rows,
                                 int cols, const float* __restrict__ norm_w,
                                 uint16_t* __restrict__ out, int64_t ld_out, int interleave) {
  griddep_wait();  // the weights may come from an earlier grid
  const int64_t n = rows * cols;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / cols;
    const int c = (int)(i % cols);
    uint16_t v;
    if (interleave) {
      const int64_t src = (r >> 7) * 64 + (r & 63);
      v = (r & 64) ? b[src * ldb + c] : a[src * lda + c];
    } else {
      v = a[r * lda + c];
    }
    if (norm_w) {
      const __nv_bfloat16 t = __float2bfloat16_rn(__uint_as_float((uint32_t)v << 16) * norm_w[c]);
      v = *reinterpret_cast<const uint16_t*>(&t);
    }
    out[r * ld_out + c] = v;
  }
}

int launch_pack_rows(const tg_bf16* a, int64_t lda, const tg_bf16* b, int64_t ldb, int64_t rows,
                     int cols, const float* norm_w, tg_bf16* out, int64_t ld_out, int interleave,
                     cudaStream_t stream) {
  const int64_t n = rows * cols;
  int64_t grid = (n + 255) / 256;
  if (grid > 8 * (int64_t)sm_count()) grid = 8 * (int64_t)sm_count();
  return launch(pack_rows_kernel, dim3((unsigned)grid), dim3(256), 0, stream,
                reinterpret_cast<const uint16_t*>(a), lda, reinterpret_cast<const uint16_t*>(b),
                ldb, rows, cols, norm_w, reinterpret_cast<uint16_t*>(out), ld_out, interleave);
}

}  // namespace tg

using namespace tg;

extern "C" int tg_linear(const tg_bf16* a, int64_t lda, const tg_bf16* w, int64_t ldw, tg_bf16* c,
                         int64_t ldc, int64_t M, int N, int K, int rmsnorm_a, float eps,
                         const tg_bf16* residual, int64_t ld_res, float* row_ssq_out,
                         int64_t ld_ssq_out, void* workspace, size_t workspace_bytes,
                         uint32_t* status, tg_stream_t stream) {
  if (M < 0 || N <= 0 || K <= 0 || (N % 128) || (K % 64)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (M == 0) return TG_OK;
  if (!a || !w || !c) return TG_ERR_INVALID_ARGUMENT;
  if (lda < K || ldw < K || ldc < N || (residual && ld_res < N)) return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(a) || !aligned16(w) || !aligned16(c) || (residual && !aligned16(residual)) ||
      !stride_ok(lda, 2) || !stride_ok(ldw, 2) || !stride_ok(ldc, 2) ||
      (residual && !stride_ok(ld_res, 2)))
    return TG_ERR_MISALIGNED;
  if (rmsnorm_a && !(eps >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (row_ssq_out && ld_ssq_out < N / 128) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());

  // CTA-pair kernel for 256-column tiles without an in-kernel norm; else one CTA per tile
  const bool pair = !rmsnorm_a && (N % 256) == 0;
  if (pair) {
    PairJob j;
    TG_TRY(out_proj_job(j, a, lda, w, ldw, c, ldc, M, N, K, residual, ld_res, row_ssq_out,
                        ld_ssq_out, status));
    return launch_pair<kPairStages, EpiStore>(j.maps, j.p, (cudaStream_t)stream, workspace,
                                              workspace_bytes);
  }
  const int bn = pick_bn(M, N);
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
  p.row_ssq_out = row_ssq_out;
  p.ld_ssq_out = ld_ssq_out;
  p.status = status;
  if (bn == 256) return launch_gemm<256, 4, EpiStore>(ta, tb, p, (cudaStream_t)stream);
  return launch_gemm<128, 3, EpiStore>(ta, tb, p, (cudaStream_t)stream);
}

static int qkv_rope_cache_impl(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv,
                               int64_t ld_w, int64_t M, int hidden, int n_q_heads,
                               int n_kv_heads, int head_dim, float eps, const int32_t* pos,
                               const float* cos_sin, int max_pos, tg_bf16* q_out, int64_t ld_q,
                               tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache,
                               int64_t slot_offset, const float* row_ssq_in, int64_t ld_ssq_in,
                               const float* q_norm_w, const float* k_norm_w, void* workspace,
                               size_t workspace_bytes, uint32_t* status, tg_stream_t stream) {
  if (head_dim != 128 || n_q_heads <= 0 || n_kv_heads <= 0 || hidden <= 0 || (hidden % 64))
    return TG_ERR_UNSUPPORTED_SHAPE;
  if (M < 0 || slot_offset < 0 || max_pos <= 0) return TG_ERR_INVALID_ARGUMENT;
  if (!pos && max_pos < M) return TG_ERR_INVALID_ARGUMENT;  // per-row table: row stride
  if (M == 0) return TG_OK;
  const int q_cols = n_q_heads * head_dim, kv_cols = n_kv_heads * head_dim;
  const int N = q_cols + 2 * kv_cols;
  if (!x || !w_qkv || !cos_sin || !q_out || !cache_k || !cache_v)
    return TG_ERR_INVALID_ARGUMENT;
  if (ld_x < hidden || ld_w < hidden || ld_q < q_cols || ld_cache < kv_cols)
    return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_qkv) || !aligned16(q_out) || !aligned16(cache_k) ||
      !aligned16(cache_v) || !aligned16(cos_sin) || !stride_ok(ld_x, 2) || !stride_ok(ld_w, 2) ||
      !stride_ok(ld_q, 2) || !stride_ok(ld_cache, 2))
    return TG_ERR_MISALIGNED;
  if (!(eps >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (row_ssq_in && (ld_ssq_in < hidden / 128 || (hidden % 128))) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  // 256-column tiles only when the Q/K/V boundaries fall on their edges; the CTA-pair
  // kernel when the row norms come precomputed
  const bool aligned256 = (q_cols % 256) == 0 && (kv_cols % 256) == 0;
  const bool pair = row_ssq_in && aligned256;
  if (q_norm_w || k_norm_w) {  // QK-norm lives in the CTA-pair kernel's epilogue only
    if (!q_norm_w || !k_norm_w || !row_ssq_in) return TG_ERR_INVALID_ARGUMENT;
    if (!aligned256) return TG_ERR_UNSUPPORTED_SHAPE;
  }
  if (pair) {
    PairJob j;
    TG_TRY(qkv_job(j, x, ld_x, w_qkv, ld_w, M, hidden, q_cols, kv_cols, eps, pos, cos_sin, max_pos,
                   q_out, ld_q, cache_k, cache_v, ld_cache, slot_offset, row_ssq_in, ld_ssq_in,
                   status, q_norm_w, k_norm_w));
    if (q_norm_w)
      return launch_pair<kPairStages, EpiQKVNorm>(j.maps, j.p, (cudaStream_t)stream, workspace,
                                                  workspace_bytes);
    return launch_pair<kPairStages, EpiQKV>(j.maps, j.p, (cudaStream_t)stream, workspace,
                                            workspace_bytes);
  }
  int bn = pick_bn(M, N);
  if (bn == 256 && !aligned256) bn = 128;
  CUtensorMap ta, tb;
  TG_TRY(make_tmap_bf16_2d(&ta, x, (uint64_t)M, (uint64_t)hidden, (uint64_t)ld_x, 64, 128));
  TG_TRY(make_tmap_bf16_2d(&tb, w_qkv, (uint64_t)N, (uint64_t)hidden, (uint64_t)ld_w, 64, bn));
  GemmParams p{};
  p.M = M;
  p.N = N;
  p.K = hidden;
  p.rmsnorm = 1;
  p.eps = eps;
  p.c = reinterpret_cast<uint16_t*>(q_out);
  p.ldc = ld_q;
  p.pos = pos;
  p.cos_sin = cos_sin;
  p.max_pos = max_pos;
  p.q_cols = q_cols;
  p.k_cols = kv_cols;
  p.k_out = reinterpret_cast<uint16_t*>(cache_k) + slot_offset * ld_cache;
  p.v_out = reinterpret_cast<uint16_t*>(cache_v) + slot_offset * ld_cache;
  p.ld_kv = ld_cache;
  p.row_ssq_in = row_ssq_in;
  p.ld_ssq_in = ld_ssq_in;
  p.status = status;
  if (bn == 256) return launch_gemm<256, 4, EpiQKV>(ta, tb, p, (cudaStream_t)stream);
  return launch_gemm<128, 3, EpiQKV>(ta, tb, p, (cudaStream_t)stream);
}

extern "C" int tg_qkv_rope_cache(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv, int64_t ld_w,
                                 int64_t M, int hidden, int n_q_heads, int n_kv_heads,
                                 int head_dim, float eps, const int32_t* pos,
                                 const float* cos_sin, int max_pos, tg_bf16* q_out, int64_t ld_q,
                                 tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache,
                                 int64_t slot_offset, const float* row_ssq_in,
                                 int64_t ld_ssq_in, void* workspace, size_t workspace_bytes,
                                 uint32_t* status, tg_stream_t stream) {
  return qkv_rope_cache_impl(x, ld_x, w_qkv, ld_w, M, hidden, n_q_heads, n_kv_heads, head_dim,
                             eps, pos, cos_sin, max_pos, q_out, ld_q, cache_k, cache_v, ld_cache,
                             slot_offset, row_ssq_in, ld_ssq_in, nullptr, nullptr, workspace,
                             workspace_bytes, status, stream);
}

extern "C" int tg_qkv_qknorm_rope_cache(
    const tg_bf16* x, int64_t ld_x, const tg_bf16* w_qkv, int64_t ld_w, int64_t M, int hidden,
    int n_q_heads, int n_kv_heads, int head_dim, float eps, const float* q_norm_w,
    const float* k_norm_w, const int32_t* pos, const float* cos_sin, int max_pos, tg_bf16* q_out,
    int64_t ld_q, tg_bf16* cache_k, tg_bf16* cache_v, int64_t ld_cache, int64_t slot_offset,
    const float* row_ssq_in, int64_t ld_ssq_in, void* workspace, size_t workspace_bytes,
    uint32_t* status, tg_stream_t stream) {
  if (!q_norm_w || !k_norm_w || !row_ssq_in) return TG_ERR_INVALID_ARGUMENT;
  return qkv_rope_cache_impl(x, ld_x, w_qkv, ld_w, M, hidden, n_q_heads, n_kv_heads, head_dim,
                             eps, pos, cos_sin, max_pos, q_out, ld_q, cache_k, cache_v, ld_cache,
                             slot_offset, row_ssq_in, ld_ssq_in, q_norm_w, k_norm_w, workspace,
                             workspace_bytes, status, stream);
}

extern "C" size_t tg_gemm_workspace_size(void) {
  return split_workspace_bytes(std::max(1, sm_count() / 2));
}

extern "C" int tg_swiglu(const tg_bf16* x, int64_t ld_x, const tg_bf16* w_gu, int64_t ld_w,
                         int64_t M, int hidden, int ffn, float eps, const float* row_ssq_in,
                         int64_t ld_ssq_in, tg_bf16* h_out, int64_t ld_h, uint32_t* status,
                         tg_stream_t stream) {
  if (hidden <= 0 || (hidden % 128) || ffn <= 0 || (ffn % 128)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (M < 0) return TG_ERR_INVALID_ARGUMENT;
  if (M == 0) return TG_OK;
  if (!x || !w_gu || !row_ssq_in || !h_out) return TG_ERR_INVALID_ARGUMENT;
  if (ld_x < hidden || ld_w < hidden || ld_h < ffn || ld_ssq_in < hidden / 128)
    return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(x) || !aligned16(w_gu) || !aligned16(h_out) || !stride_ok(ld_x, 2) ||
      !stride_ok(ld_w, 2) || !stride_ok(ld_h, 2))
    return TG_ERR_MISALIGNED;
  if (!(eps >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  PairJob j;
  TG_TRY(swiglu_job(j, x, ld_x, w_gu, ld_w, M, hidden, ffn, eps, row_ssq_in, ld_ssq_in, h_out,
                    ld_h, status));
  return launch_pair<kPairStages, EpiSwiGLU>(j.maps, j.p, (cudaStream_t)stream);
}

extern "C" int tg_fold_norm_weight(const tg_bf16* w, int64_t ld_w, int64_t rows, int cols,
                                   const float* norm_w, tg_bf16* out, int64_t ld_out,
                                   tg_stream_t stream) {
  if (rows < 0 || cols <= 0) return TG_ERR_INVALID_ARGUMENT;
  if (rows == 0) return TG_OK;
  if (!w || !norm_w || !out || ld_w < cols || ld_out < cols) return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  return launch_pack_rows(w, ld_w, nullptr, 0, rows, cols, norm_w, out, ld_out, 0,
                          (cudaStream_t)stream);
}

extern "C" int tg_pack_gate_up(const tg_bf16* w_gate, int64_t ld_gate, const tg_bf16* w_up,
                               int64_t ld_up, int ffn, int hidden, const float* norm_w,
                               tg_bf16* out, int64_t ld_out, tg_stream_t stream) {
  if (ffn <= 0 || (ffn % 64) || hidden <= 0) return TG_ERR_UNSUPPORTED_SHAPE;
  if (!w_gate || !w_up || !out || ld_gate < hidden || ld_up < hidden || ld_out < hidden)
    return TG_ERR_INVALID_ARGUMENT;
  TG_TRY(check_device());
  return launch_pack_rows(w_gate, ld_gate, w_up, ld_up, 2 * (int64_t)ffn, hidden, norm_w, out,
                          ld_out, 1, (cudaStream_t)stream);
}

extern "C" size_t tg_out_proj_qkv_workspace_size(int64_t M) {
  if (M <= 0) return 0;
  return (size_t)(2 * ((M + 255) / 256)) * sizeof(int32_t);
}

extern "C" int tg_out_proj_qkv_next(
    const tg_bf16* o, int64_t ld_o, const tg_bf16* w_o, int64_t ld_wo, tg_bf16* x, int64_t ld_x,
    float* row_ssq, int64_t ld_ssq, int64_t M, int hidden, int o_cols, const tg_bf16* w_qkv,
    int64_t ld_wqkv, int n_q_heads, int n_kv_heads, int head_dim, float eps, const int32_t* pos,
    const float* cos_sin, int max_pos, tg_bf16* q_out, int64_t ld_q, tg_bf16* cache_k,
    tg_bf16* cache_v, int64_t ld_cache, int64_t slot_offset, void* workspace,
    size_t workspace_bytes, uint32_t* status, tg_stream_t stream) {
  if (head_dim != 128 || n_q_heads <= 0 || n_kv_heads <= 0 || hidden <= 0 || (hidden % 256) ||
      o_cols <= 0 || (o_cols % 64))
    return TG_ERR_UNSUPPORTED_SHAPE;
  const int q_cols = n_q_heads * head_dim, kv_cols = n_kv_heads * head_dim;
  if ((q_cols % 256) || (kv_cols % 256)) return TG_ERR_UNSUPPORTED_SHAPE;
  if (M < 0 || slot_offset < 0 || max_pos <= 0 || !(eps >= 0.f)) return TG_ERR_INVALID_ARGUMENT;
  if (!pos && max_pos < M) return TG_ERR_INVALID_ARGUMENT;  // per-row table: row stride
  if (M == 0) return TG_OK;
  if (!o || !w_o || !x || !row_ssq || !w_qkv || !cos_sin || !q_out || !cache_k ||
      !cache_v)
    return TG_ERR_INVALID_ARGUMENT;
  if (ld_o < o_cols || ld_wo < o_cols || ld_x < hidden || ld_ssq < hidden / 128 ||
      ld_wqkv < hidden || ld_q < q_cols || ld_cache < kv_cols)
    return TG_ERR_INVALID_ARGUMENT;
  if (!aligned16(o) || !aligned16(w_o) || !aligned16(x) || !aligned16(w_qkv) ||
      !aligned16(q_out) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(cos_sin) ||
      !stride_ok(ld_o, 2) || !stride_ok(ld_wo, 2) || !stride_ok(ld_x, 2) ||
      !stride_ok(ld_wqkv, 2) || !stride_ok(ld_q, 2) || !stride_ok(ld_cache, 2))
    return TG_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < tg_out_proj_qkv_workspace_size(M) ||
      (reinterpret_cast<uintptr_t>(workspace) & 3))
    return TG_ERR_WORKSPACE;
  TG_TRY(check_device());
  PairJob j0, j1;
  TG_TRY(out_proj_job(j0, o, ld_o, w_o, ld_wo, x, ld_x, M, hidden, o_cols, x, ld_x, row_ssq,
                      ld_ssq, status));
  TG_TRY(qkv_job(j1, x, ld_x, w_qkv, ld_wqkv, M, hidden, q_cols, kv_cols, eps, pos, cos_sin,
                 max_pos, q_out, ld_q, cache_k, cache_v, ld_cache, slot_offset, row_ssq, ld_ssq,
                 status));
  const int64_t rps = (M + 255) / 256;
  int* ready = static_cast<int*>(workspace);
  // each output-projection tile of a row pair counts 4 (two epilogue groups per CTA)
  const PairChain chain{ready, ready + rps, 4 * (hidden / 256)};
  return launch_pair_chain<kPairStages, EpiStore, EpiQKV>(j0, j1, chain, (cudaStream_t)stream);
}
