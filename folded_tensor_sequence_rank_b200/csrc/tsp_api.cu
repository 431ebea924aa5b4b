// tsp_api.cu - the C ABI (include/tsp.h): argument checks, workspace layout,
// TMA tensor maps and the launch sequence of one TSP rank's layer forward.
//
// Launch sequence of tsp_rank_step (one stream, no host synchronisation):
//   LN1(x_local) -> QKV GEMM (Q local; K, V to their global rows) ->
//   attention -> O GEMM (+x, fp32 Y1) -> LN2(Y1) -> W1 GEMM (+GELU) ->
//   W2 GEMM (+Y1) -> y_local.
// The TSP exchanges (zubnet.ai news item, paragraph 2: shard broadcast, K/V
// all-gather, MLP ring) are shard pointers already resident on this GPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <nvtx3/nvToolsExt.h>

#include <cstdio>
#include <cstring>
#include <mutex>

#include "tsp.h"
#include "attn_bwd_sm100.cuh"
#include "attn_sm100.cuh"
#include "gemm_pair_sm100.cuh"
#include "gemm_sm100.cuh"
#include "misc_kernels.cuh"

// File-scope scratch of tsp_kv_project_noalloc (see noalloc_scratch below).
static __device__ __align__(256) uint8_t g_noalloc_scratch[size_t(64) << 20];

namespace {

using namespace tsp;

// NVTX range for the lifetime of a scope: every entry point and every launch
// step is named in an Nsight timeline.  Without a tool attached, a push/pop
// pair is a call through a no-op function pointer.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define TSP_CONCAT2(a, b) a##b
#define TSP_CONCAT(a, b) TSP_CONCAT2(a, b)
#define TSP_RANGE(name) NvtxRange TSP_CONCAT(tsp_nvtx_range_, __LINE__)(name)

constexpr uint64_t kDefaultTimeoutNs = 2000000000ull;  // 2 s per wait
constexpr size_t kAlign = 1024;

thread_local char g_cuda_err[256] = "";

int cuda_fail(cudaError_t e, const char* where) {
  std::snprintf(g_cuda_err, sizeof(g_cuda_err), "%s: %s", where, cudaGetErrorString(e));
  return TSP_ERR_CUDA;
}

#define TSP_CUDA(call)                                   \
  do {                                                   \
    cudaError_t e_ = (call);                             \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call);  \
  } while (0)

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ---------------------------------------------------------------- tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D fp16 (or bf16) row-major [rows, cols] with row stride ld elements;
// box = 64 columns (128 bytes, 128B swizzle) x box_rows rows.
int make_map(CUtensorMap* m, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows,
             bool bf16 = false) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled unavailable");
    return TSP_ERR_CUDA;
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return TSP_ERR_CUDA;
  }
  return TSP_OK;
}

// 2-D fp32 row-major [rows, cols] with row stride ld elements; box = box_cols
// (<= 32: at most 128 bytes, 128B swizzle) x box_rows rows.  Used as the
// destination of bulk reductions.
int make_map_f32(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows, int box_cols) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled unavailable");
    return TSP_ERR_CUDA;
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled (fp32) failed (%d)", static_cast<int>(r));
    return TSP_ERR_CUDA;
  }
  return TSP_OK;
}

// The output of a residual epilogue as the destination of tensor stores:
// [rows, cols] row-major with row stride ld elements, fp32 (32 x 32 boxes of
// 128-byte rows, 128B swizzle) or bf16 (32 x 32 boxes of 64-byte rows, 64B
// swizzle).
int make_map_store(CUtensorMap* m, void* base, int64_t rows, int64_t cols, int64_t ld, bool f32) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled unavailable");
    return TSP_ERR_CUDA;
  }
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * (f32 ? 4 : 2)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "cuTensorMapEncodeTiled (store) failed (%d)", static_cast<int>(r));
    return TSP_ERR_CUDA;
  }
  return TSP_OK;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// ---------------------------------------------------------------- sizes
struct Sizes {
  int64_t T, c, L;
  int64_t c_pad;  // c rounded up to a whole 128-row tile (rows of the per-chunk stashes)
  int h, H, d, F, D, hs, Fs;
};

Sizes sizes_of(const tsp_dims* dims, int D) {
  Sizes s;
  s.T = dims->T;
  s.D = D;
  s.c = dims->T / (2 * D);
  s.c_pad = (s.c + 127) / 128 * 128;
  s.L = 2 * s.c;
  s.h = dims->h;
  s.H = dims->n_heads;
  s.d = dims->head_dim;
  s.F = dims->ffn;
  s.hs = dims->h / D;
  s.Fs = dims->ffn / D;
  return s;
}

struct WsLayout {
  size_t status, xn, q, a, y1, hbuf, counters, lse, total;
};

// Bytes of a per-head, per-chunk fp32 stash [H][2][c_pad].
size_t stash_bytes(const Sizes& s) { return static_cast<size_t>(s.H) * 2 * s.c_pad * 4; }

WsLayout ws_layout(const Sizes& s) {
  WsLayout w;
  size_t o = 0;
  w.status = o; o += align_up(256);
  w.counters = o; o += align_up(256);
  w.xn = o; o += align_up(static_cast<size_t>(s.L) * s.h * 2);
  w.q = o; o += align_up(static_cast<size_t>(s.L) * s.h * 2);
  w.a = o; o += align_up(static_cast<size_t>(s.L) * s.h * 2);
  w.y1 = o; o += align_up(static_cast<size_t>(s.L) * s.h * 4);
  w.hbuf = o; o += align_up(static_cast<size_t>(s.L) * s.F * 2);
  w.lse = o; o += align_up(stash_bytes(s));
  w.total = o;
  return w;
}

// Workspace of tsp_attn_backward: status section, work-queue counter, Delta.
struct AbwdLayout {
  size_t status, counters, delta, total;
};

AbwdLayout abwd_layout(const Sizes& s) {
  AbwdLayout b;
  size_t o = 0;
  b.status = o; o += align_up(256);
  b.counters = o; o += align_up(256);
  b.delta = o; o += align_up(stash_bytes(s));
  b.total = o;
  return b;
}

int check_dims(const tsp_dims* dims, int D) {
  if (!dims) return TSP_ERR_INVALID_ARG;
  if (D < 1 || D > TSP_MAX_D) return D < 1 ? TSP_ERR_INVALID_ARG : TSP_ERR_UNSUPPORTED;
  if (dims->T < 0 || dims->h <= 0 || dims->n_heads <= 0 || dims->head_dim <= 0 || dims->ffn <= 0)
    return TSP_ERR_INVALID_ARG;
  if (dims->T % (2 * D) != 0) return TSP_ERR_INVALID_ARG;
  if (dims->n_heads % D != 0 || dims->ffn % D != 0) return TSP_ERR_INVALID_ARG;
  if (static_cast<int64_t>(dims->n_heads) * dims->head_dim != dims->h) return TSP_ERR_INVALID_ARG;
  if (!(dims->ln_eps >= 0.f) || !(dims->softmax_scale > 0.f)) return TSP_ERR_INVALID_ARG;
  if (dims->T >= (int64_t(1) << 31)) return TSP_ERR_UNSUPPORTED;
  if (dims->head_dim != 64 && dims->head_dim != 128) return TSP_ERR_UNSUPPORTED;
  // h <= 8192: the LayerNorm kernels (forward and backward) hold a row as at
  // most 8 groups of 4 values per thread of a 256-thread block
  if (dims->h % 64 != 0 || dims->h > 8192) return TSP_ERR_UNSUPPORTED;
  if ((dims->h / D) % 64 != 0 || (dims->ffn / D) % 64 != 0) return TSP_ERR_UNSUPPORTED;
  return TSP_OK;
}

int check_weights(const tsp_weights* w, int D) {
  if (!w || w->D != D) return TSP_ERR_INVALID_ARG;
  for (int k = 0; k < D; ++k) {
    const void* ps[6] = {w->wq[k], w->wk[k], w->wv[k], w->wo[k], w->w1[k], w->w2[k]};
    for (const void* p : ps)
      if (!p || !aligned16(p)) return TSP_ERR_INVALID_ARG;
  }
  return TSP_OK;
}

// ---------------------------------------------------------------- launches
template <typename Tin>
int launch_layernorm(const Tin* x, __half* y, int64_t rows, int h, float eps, cudaStream_t st) {
  TSP_RANGE("layernorm");
  if (rows == 0) return TSP_OK;
  if (h >= 1024 && h <= 8192) {  // one row per block
    const dim3 grid(static_cast<unsigned>(rows));
    const int g = (h + 1023) / 1024;
    if (g <= 1) layernorm_block_kernel<Tin, 1><<<grid, 256, 0, st>>>(x, y, h, eps);
    else if (g <= 2) layernorm_block_kernel<Tin, 2><<<grid, 256, 0, st>>>(x, y, h, eps);
    else if (g <= 4) layernorm_block_kernel<Tin, 4><<<grid, 256, 0, st>>>(x, y, h, eps);
    else layernorm_block_kernel<Tin, 8><<<grid, 256, 0, st>>>(x, y, h, eps);
    TSP_CUDA(cudaGetLastError());
    return TSP_OK;
  }
  const int warps = 8;
  const dim3 grid(static_cast<unsigned>((rows + warps - 1) / warps));
  const int nch = h / 8;
  const int maxc = (nch + 31) / 32;
  if (maxc <= 1) layernorm_rows_kernel<Tin, 1><<<grid, 256, 0, st>>>(x, y, rows, h, eps);
  else if (maxc <= 2) layernorm_rows_kernel<Tin, 2><<<grid, 256, 0, st>>>(x, y, rows, h, eps);
  else if (maxc <= 4) layernorm_rows_kernel<Tin, 4><<<grid, 256, 0, st>>>(x, y, rows, h, eps);
  else if (maxc <= 8) layernorm_rows_kernel<Tin, 8><<<grid, 256, 0, st>>>(x, y, rows, h, eps);
  else layernorm_rows_kernel<Tin, 16><<<grid, 256, 0, st>>>(x, y, rows, h, eps);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

template <int BN>
int launch_gemm_bn(GemmParams& p, cudaStream_t st) {
  using S = GemmShape<BN>;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_f16_tcgen05<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
  });
  TSP_CUDA(attr_err);
  const int tiles = ((p.M + kGemmBM - 1) / kGemmBM) * (p.N / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  gemm_f16_tcgen05<BN><<<grid, kGemmThreads, S::kSmemBytes, st>>>(p);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

// 256-column tiles run on CTA pairs (clusters of two, 256 x 256 tiles).
int launch_gemm_pair(GemmParams& p, cudaStream_t st) {
  using S = GemmPairShape;
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  static int max_clusters = 0;
  std::call_once(once, [] {
    attr_err = cudaFuncSetAttribute(gemm_pair_f16_tcgen05, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
    if (attr_err != cudaSuccess) return;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    attr_err = cudaOccupancyMaxActiveClusters(&max_clusters, gemm_pair_f16_tcgen05, &cfg);
  });
  TSP_CUDA(attr_err);
  if (max_clusters <= 0) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "no CTA pair of the GEMM kernel fits on this GPU");
    return TSP_ERR_CUDA;
  }
  // residual epilogues write through tensor stores when the output allows them
  p.tma_out = 0;
  if (p.epi == kEpiResidual && aligned16(p.out[0]) && (p.ldo * (p.out_f32 ? 4 : 2)) % 16 == 0 && p.N % 32 == 0) {
    const int rc = make_map_store(&p.map_out, p.out[0], p.M, p.N, p.ldo, p.out_f32 != 0);
    if (rc) return rc;
    p.tma_out = 1;
  }
  const int tiles = ((p.M + kPairBM - 1) / kPairBM) * (p.N / kPairBN);
  const int pairs = tiles < max_clusters ? tiles : max_clusters;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = S::kSmemBytes;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  TSP_CUDA(cudaLaunchKernelEx(&cfg, gemm_pair_f16_tcgen05, p));
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

int pick_bn(int n_block) {
  if (n_block % 256 == 0) return 256;
  if (n_block % 128 == 0) return 128;
  return 64;
}

// Rows of a B tile each CTA loads: half of a pair tile for 256 columns.
int b_box_rows(int bn) { return bn == 256 ? 128 : bn; }

int launch_gemm(GemmParams& p, int bn, cudaStream_t st) {
  TSP_RANGE("gemm");
  if (p.M == 0) return TSP_OK;
  switch (bn) {
    case 256: return launch_gemm_pair(p, st);
    case 128: return launch_gemm_bn<128>(p, st);
    default: return launch_gemm_bn<64>(p, st);
  }
}

void gemm_common(GemmParams& p, const Sizes& s, int rank, int* status) {
  p.c = static_cast<int>(s.c);
  p.off0 = static_cast<int64_t>(rank) * s.c;                 // chunk r
  p.off1 = static_cast<int64_t>(2 * s.D - 1 - rank) * s.c - s.c;  // chunk 2D-1-r
  p.remap_rows = s.T;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
}

// N-split projection of xn [L, h] by nseg weight families (each D shards
// [h/D, h]) into nseg outputs [*, h]; remap[i] sends rows to global rows.
int launch_proj(const Sizes& s, int rank, const __half* xn, const void* const* fam[3], void* out[3],
                const int remap[3], int nseg, int epi, int F_cols, int* status, cudaStream_t st,
                void* out_t = nullptr) {
  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int shard_n = F_cols / s.D;
  int rc = make_map(&p.map_a, xn, s.L, s.h, s.h, kGemmBM);
  if (rc) return rc;
  const int bn = pick_bn(shard_n);
  for (int seg = 0; seg < nseg; ++seg)
    for (int k = 0; k < s.D; ++k) {
      rc = make_map(&p.map_b[seg * s.D + k], fam[seg][k], shard_n, s.h, s.h, b_box_rows(bn));
      if (rc) return rc;
    }
  p.M = static_cast<int>(s.L);
  p.N = nseg * F_cols;
  p.K = s.h;
  p.ksplit = 0;
  p.shard_n = shard_n;
  p.shard_k = s.h;
  p.seg_n = F_cols;
  p.epi = epi;
  for (int i = 0; i < nseg; ++i) {
    p.out[i] = out[i];
    p.remap[i] = remap[i];
  }
  p.ldo = F_cols;
  if (out_t && s.L % kGemmBM) return TSP_ERR_UNSUPPORTED;  // the transposed store needs whole warps
  p.out_t = out_t;  // transposed GELU copy [N, L] (single segment, no remap)
  p.ld_t = s.L;
  gemm_common(p, s, rank, status);
  return launch_gemm(p, bn, st);
}

// launch_proj with the shard list of `shards` (its D) and the zigzag row
// mapping of `zz` (rank, D, c): one shard per segment whose K/V rows still go
// to the rank's global positions.
int launch_proj_zz(const Sizes& zz, const Sizes& shards, int rank, const __half* xn, const void* const* fam[3],
                   void* out[3], const int remap[3], int nseg, int epi, int F_cols, int* status, cudaStream_t st) {
  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int shard_n = F_cols / shards.D;
  int rc = make_map(&p.map_a, xn, zz.L, zz.h, zz.h, kGemmBM);
  if (rc) return rc;
  const int bn = pick_bn(shard_n);
  for (int seg = 0; seg < nseg; ++seg)
    for (int k = 0; k < shards.D; ++k) {
      rc = make_map(&p.map_b[seg * shards.D + k], fam[seg][k], shard_n, zz.h, zz.h, b_box_rows(bn));
      if (rc) return rc;
    }
  p.M = static_cast<int>(zz.L);
  p.N = nseg * F_cols;
  p.K = zz.h;
  p.ksplit = 0;
  p.shard_n = shard_n;
  p.shard_k = zz.h;
  p.seg_n = F_cols;
  p.epi = epi;
  for (int i = 0; i < nseg; ++i) {
    p.out[i] = out[i];
    p.remap[i] = remap[i];
  }
  p.ldo = F_cols;
  gemm_common(p, zz, rank, status);
  return launch_gemm(p, bn, st);
}

// K-split: out = resid + sum_k A[:, k-block] W_k^T, W_k [h, Kdim/D].
int launch_ksplit(const Sizes& s, int rank, const __half* a, int Kdim, const void* const* fam, const void* resid,
                  int resid_f32, void* out, int out_f32, int* status, cudaStream_t st) {
  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int shard_k = Kdim / s.D;
  const int bn = pick_bn(s.h);
  int rc = make_map(&p.map_a, a, s.L, Kdim, Kdim, kGemmBM);
  if (rc) return rc;
  for (int k = 0; k < s.D; ++k) {
    rc = make_map(&p.map_b[k], fam[k], s.h, shard_k, shard_k, b_box_rows(bn));
    if (rc) return rc;
  }
  p.M = static_cast<int>(s.L);
  p.N = s.h;
  p.K = Kdim;
  p.ksplit = 1;
  p.shard_n = s.h;
  p.shard_k = shard_k;
  p.seg_n = s.h;
  p.epi = kEpiResidual;
  p.out[0] = out;
  p.ldo = s.h;
  p.resid = resid;
  p.resid_f32 = resid_f32;
  p.out_f32 = out_f32;
  gemm_common(p, s, rank, status);
  return launch_gemm(p, bn, st);
}

template <int HD>
cudaError_t prepare_attention() {
  return cudaFuncSetAttribute(attn_fwd_tcgen05<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              AttnShape<HD>::kSmemBytes);
}

// The attention kernel re-splits its registers between warpgroups
// (setmaxnreg): the split adds up only for the allocation it was built for;
// with any other count an increase could wait forever, so refuse to launch.
template <typename Kernel>
int check_launch_regs(Kernel kernel, int want, int& cached) {
  if (cached < 0) {
    cudaFuncAttributes fa = {};
    TSP_CUDA(cudaFuncGetAttributes(&fa, kernel));
    cached = fa.numRegs;
  }
  if (cached != want) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err), "kernel built with %d registers per thread, not %d", cached, want);
    return TSP_ERR_CUDA;
  }
  return TSP_OK;
}

template <int HD>
int check_attention_regs() {
  static int regs = -1;
  return check_launch_regs(attn_fwd_tcgen05<HD>, kAttnLaunchRegs, regs);
}

int launch_attention(const Sizes& s, int rank, const tsp_dims* dims, const __half* q, const void* k_full,
                     const void* v_full, __half* out, float* lse, int* counter, int* status, cudaStream_t st) {
  TSP_RANGE("attention");
  if (s.L == 0) return TSP_OK;
  static thread_local AttnParams p;
  std::memset(&p, 0, sizeof(p));
  int rc = make_map(&p.map_q, q, s.L, s.h, s.h, kAttnBM);
  if (rc) return rc;
  rc = make_map(&p.map_k, k_full, s.T, s.h, s.h, kAttnBN);
  if (rc) return rc;
  rc = make_map(&p.map_v, v_full, s.T, s.h, s.h, kAttnBN);
  if (rc) return rc;
  p.out = out;
  p.ldo = s.h;
  p.c = static_cast<int>(s.c);
  p.rank = rank;
  p.D = s.D;
  p.H = s.H;
  p.nqt = static_cast<int>((s.c + kAttnBM - 1) / kAttnBM);
  p.npairs = (p.nqt + 1) / 2;
  p.n_items = 2 * p.npairs * s.H;
  p.scale_log2 = dims->softmax_scale * 1.4426950408889634f;
  p.counter = counter;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  p.lse = lse;
  p.c_pad = static_cast<int>(s.c_pad);
  p.q = q;
  p.k = static_cast<const __half*>(k_full);
  p.ldqk = s.h;
  TSP_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  if (s.d == 128) {
    static std::once_flag once;
    static cudaError_t e = cudaSuccess;
    std::call_once(once, [] { e = prepare_attention<128>(); });
    TSP_CUDA(e);
    if ((rc = check_attention_regs<128>())) return rc;
    attn_fwd_tcgen05<128><<<grid, kAttnThreads, AttnShape<128>::kSmemBytes, st>>>(p);
  } else {
    static std::once_flag once;
    static cudaError_t e = cudaSuccess;
    std::call_once(once, [] { e = prepare_attention<64>(); });
    TSP_CUDA(e);
    if ((rc = check_attention_regs<64>())) return rc;
    attn_fwd_tcgen05<64><<<grid, kAttnThreads, AttnShape<64>::kSmemBytes, st>>>(p);
  }
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

struct Ctx {
  Sizes s;
  WsLayout lay;
  uint8_t* ws;
  int* status;
  int* counters;
  __half *xn, *q, *a, *hbuf;
  float *y1, *lse;
};

int make_ctx(Ctx& c, const tsp_dims* dims, const tsp_weights* w, int rank, void* ws, size_t ws_bytes) {
  int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  rc = check_weights(w, D);
  if (rc) return rc;
  if (rank < 0 || rank >= D) return TSP_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  c.s = sizes_of(dims, D);
  c.lay = ws_layout(c.s);
  if (ws_bytes < c.lay.total) return TSP_ERR_WORKSPACE;
  c.ws = static_cast<uint8_t*>(ws);
  c.status = reinterpret_cast<int*>(c.ws + c.lay.status);
  c.counters = reinterpret_cast<int*>(c.ws + c.lay.counters);
  c.xn = reinterpret_cast<__half*>(c.ws + c.lay.xn);
  c.q = reinterpret_cast<__half*>(c.ws + c.lay.q);
  c.a = reinterpret_cast<__half*>(c.ws + c.lay.a);
  c.y1 = reinterpret_cast<float*>(c.ws + c.lay.y1);
  c.hbuf = reinterpret_cast<__half*>(c.ws + c.lay.hbuf);
  c.lse = reinterpret_cast<float*>(c.ws + c.lay.lse);
  return TSP_OK;
}

int record(cudaEvent_t* ev, int i, cudaStream_t st) {
  if (ev) TSP_CUDA(cudaEventRecord(ev[i], st));
  return TSP_OK;
}

// Everything after the projections: attention, O, LN2, W1, W2.
int layer_tail(Ctx& c, const tsp_dims* dims, const tsp_weights* w, int rank, const void* x_local, const void* k_full,
               const void* v_full, void* y_local, int y_dtype, cudaStream_t st, cudaEvent_t* ev) {
  const Sizes& s = c.s;
  int rc = launch_attention(s, rank, dims, c.q, k_full, v_full, c.a, c.lse, c.counters, c.status, st);
  if (rc) return rc;
  if ((rc = record(ev, 3, st))) return rc;
  rc = launch_ksplit(s, rank, c.a, s.h, reinterpret_cast<const void* const*>(w->wo), x_local, 0, c.y1, 1, c.status, st);
  if (rc) return rc;
  if ((rc = record(ev, 4, st))) return rc;
  rc = launch_layernorm<float>(c.y1, c.xn, s.L, s.h, dims->ln_eps, st);
  if (rc) return rc;
  if ((rc = record(ev, 5, st))) return rc;
  const void* const* w1fam[3] = {reinterpret_cast<const void* const*>(w->w1), nullptr, nullptr};
  void* hout[3] = {c.hbuf, nullptr, nullptr};
  const int noremap[3] = {0, 0, 0};
  rc = launch_proj(s, rank, c.xn, w1fam, hout, noremap, 1, kEpiGeluF16, s.F, c.status, st);
  if (rc) return rc;
  if ((rc = record(ev, 6, st))) return rc;
  rc = launch_ksplit(s, rank, c.hbuf, s.F, reinterpret_cast<const void* const*>(w->w2), c.y1, 1, y_local,
                     y_dtype == TSP_OUT_F32, c.status, st);
  if (rc) return rc;
  return record(ev, 7, st);
}

// ---------------------------------------------------------------- attention backward
template <int HD>
int launch_attn_bwd_hd(AttnBwdParams& p, cudaStream_t st) {
  using S = AttnBwdShape<HD>;
  static std::once_flag once;
  static cudaError_t e = cudaSuccess;
  std::call_once(once, [] {
    e = cudaFuncSetAttribute(attn_bwd_tcgen05<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kSmemBytes);
  });
  TSP_CUDA(e);
  // the kernel re-splits its registers (setmaxnreg) for this launch allocation
  static int regs = -1;
  const int rc = check_launch_regs(attn_bwd_tcgen05<HD>, kBwdLaunchRegs, regs);
  if (rc) return rc;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  attn_bwd_tcgen05<HD><<<grid, kBwdThreads, S::kSmemBytes, st>>>(p);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

// Delta, then the key-tile-outer backward kernel.  dq is zeroed here (the
// kernel adds every key tile's contribution); dk, dv are added to.
int launch_attn_backward(const Sizes& s, int rank, const tsp_dims* dims, const __half* q, const void* k_full,
                         const void* v_full, const __half* o, const float* lse, const __half* d_o, float* dq,
                         float* dk, float* dv, float* delta, int* counter, int* status, cudaStream_t st) {
  TSP_RANGE("attention_backward");
  if (s.L == 0) return TSP_OK;
  TSP_CUDA(cudaMemsetAsync(dq, 0, static_cast<size_t>(s.L) * s.h * 4, st));
  const dim3 grid_rows(static_cast<unsigned>(s.L));
  if (s.d == 128)
    attn_bwd_delta_kernel<128><<<grid_rows, 256, 0, st>>>(d_o, o, delta, s.h, static_cast<int>(s.c),
                                                          static_cast<int>(s.c_pad), dims->softmax_scale);
  else
    attn_bwd_delta_kernel<64><<<grid_rows, 256, 0, st>>>(d_o, o, delta, s.h, static_cast<int>(s.c),
                                                         static_cast<int>(s.c_pad), dims->softmax_scale);
  TSP_CUDA(cudaGetLastError());
  static thread_local AttnBwdParams p;
  std::memset(&p, 0, sizeof(p));
  int rc = make_map(&p.map_q, q, s.L, s.h, s.h, kBwdTile);
  if (rc) return rc;
  if ((rc = make_map(&p.map_do, d_o, s.L, s.h, s.h, kBwdTile))) return rc;
  if ((rc = make_map(&p.map_k, k_full, s.T, s.h, s.h, kBwdTile))) return rc;
  if ((rc = make_map(&p.map_v, v_full, s.T, s.h, s.h, kBwdTile))) return rc;
  if ((rc = make_map_f32(&p.map_dq, dq, s.L, s.h, s.h, 32, 32))) return rc;
  p.lse = lse;
  p.delta = delta;
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.ld = s.h;
  p.T = s.T;
  p.c = static_cast<int>(s.c);
  p.c_pad = static_cast<int>(s.c_pad);
  p.rank = rank;
  p.D = s.D;
  p.H = s.H;
  p.nqt = static_cast<int>((s.c + kBwdTile - 1) / kBwdTile);
  const int64_t last = (2 * s.D - rank) * s.c;  // last position of the rank + 1
  p.nkt = static_cast<int>((last + kBwdTile - 1) / kBwdTile);
  p.n_items = p.nkt * s.H;
  p.scale_log2 = dims->softmax_scale * 1.4426950408889634f;
  p.scale = dims->softmax_scale;
  p.counter = counter;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  TSP_CUDA(cudaMemsetAsync(counter, 0, sizeof(int), st));
  return s.d == 128 ? launch_attn_bwd_hd<128>(p, st) : launch_attn_bwd_hd<64>(p, st);
}

// ---------------------------------------------------------------- MLP backward
struct BwdLayout {
  size_t status, xn2, u, du, dxn2, xn2t, dut, ht, dyt, total;
};

BwdLayout bwd_layout(const Sizes& s) {
  BwdLayout b;
  const size_t Lh = static_cast<size_t>(s.L) * s.h, LF = static_cast<size_t>(s.L) * s.F;
  size_t o = 0;
  b.status = o; o += align_up(256);
  b.xn2 = o; o += align_up(Lh * 2);
  b.u = o; o += align_up(LF * 2);
  b.du = o; o += align_up(LF * 2);
  b.dxn2 = o; o += align_up(Lh * 4);
  b.xn2t = o; o += align_up(Lh * 2);
  b.dut = o; o += align_up(LF * 2);
  b.ht = o; o += align_up(LF * 2);
  b.dyt = o; o += align_up(Lh * 2);
  b.total = o;
  return b;
}

// C [M, N] = A [M, K] * B [N, K]^T with one B map: A and B K-major with row
// strides lda / ldb, both fp16 or both bf16; epilogue kEpiStoreF32 (out fp32)
// or kEpiGeluBwd (out bf16, aux = U fp16), row stride ldo.
int launch_plain(const void* a, int M, int K, int64_t lda, const void* b, int N, int64_t ldb, bool bf16, int epi,
                 void* out, int64_t ldo, const void* aux, int* status, cudaStream_t st, void* out_t = nullptr,
                 int64_t ld_t = 0) {
  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int bn = pick_bn(N);
  int rc = make_map(&p.map_a, a, M, K, lda, kGemmBM, bf16);
  if (rc) return rc;
  rc = make_map(&p.map_b[0], b, N, K, ldb, b_box_rows(bn), bf16);
  if (rc) return rc;
  p.M = M;
  p.N = N;
  p.K = K;
  p.ksplit = 0;
  p.shard_n = N;
  p.shard_k = K;
  p.seg_n = N;
  p.epi = epi;
  p.fmt_bf16 = bf16 ? 1 : 0;
  p.out[0] = out;
  p.ldo = ldo;
  p.resid = aux;
  if (out_t && M % kGemmBM) return TSP_ERR_UNSUPPORTED;  // the transposed store needs whole warps
  p.out_t = out_t;
  p.ld_t = ld_t;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  return launch_gemm(p, bn, st);
}

template <typename Tin>
int launch_transpose(const Tin* in, int64_t rows, int cols, __nv_bfloat16* out, cudaStream_t st) {
  TSP_RANGE("transpose");
  if (rows == 0) return TSP_OK;
  if (rows % 8 || cols % 8) return TSP_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>((rows + 63) / 64), static_cast<unsigned>((cols + 63) / 64));
  transpose_bf16_kernel<Tin><<<grid, 256, 0, st>>>(in, rows, cols, out);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

template <typename Tx, typename Tr>
int launch_ln_backward(const Tx* y1, const float* g, const Tr* dy, float* dy1, __nv_bfloat16* dy1_bf16, int64_t rows,
                       int h, float eps, cudaStream_t st) {
  TSP_RANGE("layernorm_backward");
  if (rows == 0) return TSP_OK;
  const int groups = (h + 1023) / 1024;  // groups of 4 values per thread
  const dim3 grid(static_cast<unsigned>(rows));
  if (groups <= 1) ln_backward_rows_kernel<4, Tx, Tr><<<grid, 256, 0, st>>>(y1, g, dy, dy1, dy1_bf16, h, eps);
  else if (groups <= 2) ln_backward_rows_kernel<8, Tx, Tr><<<grid, 256, 0, st>>>(y1, g, dy, dy1, dy1_bf16, h, eps);
  else if (groups <= 4) ln_backward_rows_kernel<16, Tx, Tr><<<grid, 256, 0, st>>>(y1, g, dy, dy1, dy1_bf16, h, eps);
  else ln_backward_rows_kernel<32, Tx, Tr><<<grid, 256, 0, st>>>(y1, g, dy, dy1, dy1_bf16, h, eps);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

int launch_convert_bf16(const float* in, __nv_bfloat16* out, int64_t n, cudaStream_t st) {
  if (n == 0) return TSP_OK;
  const int64_t threads = n / 8;
  convert_bf16_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, st>>>(in, out, n);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

// Shapes the backward implements: whole 256-column tiles, and whole 128-row
// tiles of tokens (the transposed epilogue stores need every lane of a warp).
int check_backward_shape(const Sizes& s) {
  if (s.h % 256 || s.F % 256 || s.L % 128) return TSP_ERR_UNSUPPORTED;
  return TSP_OK;
}

// The MLP half of the backward (tsp_mlp_backward's steps): dY1 = dL/dY1 (fp32,
// and a bf16 copy when dy1b is not null), dW1, dW2.
int mlp_backward_core(const Sizes& s, const tsp_dims* dims, const tsp_weights* w, const void* w1_full,
                      const void* w2_full, const float* y1, const __nv_bfloat16* dy, float* dy1, __nv_bfloat16* dy1b,
                      float* dw1, float* dw2, uint8_t* base, const BwdLayout& b, cudaStream_t stream,
                      cudaEvent_t* ev) {
  int rc;
  int* status = reinterpret_cast<int*>(base + b.status);
  if ((rc = record(ev, 0, stream))) return rc;
  if (s.L == 0) {  // no tokens: zero weight gradients
    TSP_CUDA(cudaMemsetAsync(dw1, 0, static_cast<size_t>(s.h) * s.F * 4, stream));
    TSP_CUDA(cudaMemsetAsync(dw2, 0, static_cast<size_t>(s.F) * s.h * 4, stream));
    for (int i = 1; i < TSP_N_STEP_EVENTS; ++i)
      if ((rc = record(ev, i, stream))) return rc;
    return TSP_OK;
  }
  __half* xn2 = reinterpret_cast<__half*>(base + b.xn2);
  __half* u = reinterpret_cast<__half*>(base + b.u);
  __nv_bfloat16* du = reinterpret_cast<__nv_bfloat16*>(base + b.du);
  float* dxn2 = reinterpret_cast<float*>(base + b.dxn2);
  __nv_bfloat16* xn2t = reinterpret_cast<__nv_bfloat16*>(base + b.xn2t);
  __nv_bfloat16* dut = reinterpret_cast<__nv_bfloat16*>(base + b.dut);
  __nv_bfloat16* ht = reinterpret_cast<__nv_bfloat16*>(base + b.ht);
  __nv_bfloat16* dyt = reinterpret_cast<__nv_bfloat16*>(base + b.dyt);
  const int L = static_cast<int>(s.L);
  // Xn2 = LN2(Y1), U = Xn2 W1 (fp16 shards, as in the forward); the same
  // epilogue writes GELU(U)^T (bf16 [F, L]) for dW2
  rc = launch_layernorm<float>(y1, xn2, s.L, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  const void* const* w1fam[3] = {reinterpret_cast<const void* const*>(w->w1), nullptr, nullptr};
  void* uout[3] = {u, nullptr, nullptr};
  const int noremap[3] = {0, 0, 0};
  rc = launch_proj(s, 0, xn2, w1fam, uout, noremap, 1, kEpiStoreF16, s.F, status, stream, ht);
  if (rc) return rc;
  if ((rc = record(ev, 1, stream))) return rc;
  // dU = (dY W2^T) * GELU'(U): B = W2 [F, h] is K-major over h; the
  // epilogue also writes dU^T (bf16 [F, L]) for dW1
  rc = launch_plain(dy, L, s.h, s.h, w2_full, s.F, s.h, true, kEpiGeluBwd, du, s.F, u, status, stream, dut, s.L);
  if (rc) return rc;
  if ((rc = record(ev, 2, stream))) return rc;
  // dXn2 = dU W1^T: B = W1 [h, F] is K-major over F
  rc = launch_plain(du, L, s.F, s.F, w1_full, s.h, s.F, true, kEpiStoreF32, dxn2, s.h, nullptr, status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 3, stream))) return rc;
  // dY1 = dY + LN2'(Y1)^T dXn2
  rc = launch_ln_backward<float, __nv_bfloat16>(y1, dxn2, dy, dy1, dy1b, s.L, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  if ((rc = record(ev, 4, stream))) return rc;
  // token-major operands of the weight gradients (reduction over the tokens)
  if ((rc = launch_transpose<__half>(xn2, s.L, s.h, xn2t, stream))) return rc;
  if ((rc = launch_transpose<__nv_bfloat16>(dy, s.L, s.h, dyt, stream))) return rc;
  if ((rc = record(ev, 5, stream))) return rc;
  // dW1 [h, F] = Xn2^T dU ; dW2 [F, h] = GELU(U)^T dY
  rc = launch_plain(xn2t, s.h, L, L, dut, s.F, L, true, kEpiStoreF32, dw1, s.F, nullptr, status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 6, stream))) return rc;
  rc = launch_plain(ht, s.F, L, L, dyt, s.h, L, true, kEpiStoreF32, dw2, s.h, nullptr, status, stream);
  if (rc) return rc;
  return record(ev, 7, stream);
}

// Workspace of tsp_layer_backward: the MLP half's (its status section first),
// then the attention half's operands.
struct LayerBwdLayout {
  BwdLayout mlp;
  size_t dy1, dy1b, dy1t, at, d_o, dq, dqb, dqt, xn1, xn1t, dxn1, counters, delta, total;
};

LayerBwdLayout lbwd_layout(const Sizes& s) {
  LayerBwdLayout l;
  l.mlp = bwd_layout(s);
  const size_t Lh = static_cast<size_t>(s.L) * s.h;
  size_t o = l.mlp.total;
  l.dy1 = o; o += align_up(Lh * 4);
  l.dy1b = o; o += align_up(Lh * 2);
  l.dy1t = o; o += align_up(Lh * 2);
  l.at = o; o += align_up(Lh * 2);
  l.d_o = o; o += align_up(Lh * 2);
  l.dq = o; o += align_up(Lh * 4);
  l.dqb = o; o += align_up(Lh * 2);
  l.dqt = o; o += align_up(Lh * 2);
  l.xn1 = o; o += align_up(Lh * 2);
  l.xn1t = o; o += align_up(Lh * 2);
  l.dxn1 = o; o += align_up(Lh * 4);
  l.counters = o; o += align_up(256);
  l.delta = o; o += align_up(stash_bytes(s));
  l.total = o;
  return l;
}

// Workspace of tsp_kv_backward.
struct KvBwdLayout {
  size_t status, xn1, xn1t, kv, kvt, dxn, total;
};

KvBwdLayout kvbwd_layout(const Sizes& s) {
  KvBwdLayout k;
  const size_t Lh = static_cast<size_t>(s.L) * s.h;
  size_t o = 0;
  k.status = o; o += align_up(256);
  k.xn1 = o; o += align_up(Lh * 2);
  k.xn1t = o; o += align_up(Lh * 2);
  k.kv = o; o += align_up(Lh * 4);
  k.kvt = o; o += align_up(Lh * 4);
  k.dxn = o; o += align_up(Lh * 4);
  k.total = o;
  return k;
}

// dXn [L, h] = [dK | dV] [Wk ; Wv]^T: A = [dK | dV] bf16 [L, 2h]; the K loop
// walks Wk (row-major [h_in, h_out]: K-major over h_out) for its first h
// columns and Wv for the next h; fp32 out.
int launch_kv_grad_input(const __nv_bfloat16* kv, int L, int h, const void* wk, const void* wv, float* out,
                         int* status, cudaStream_t st) {
  static thread_local GemmParams p;
  std::memset(&p, 0, sizeof(p));
  const int bn = pick_bn(h);
  int rc = make_map(&p.map_a, kv, L, 2 * h, 2 * h, kGemmBM, true);
  if (rc) return rc;
  if ((rc = make_map(&p.map_b[0], wk, h, h, h, b_box_rows(bn), true))) return rc;
  if ((rc = make_map(&p.map_b[1], wv, h, h, h, b_box_rows(bn), true))) return rc;
  p.M = L;
  p.N = h;
  p.K = 2 * h;
  p.ksplit = 1;
  p.shard_n = h;
  p.shard_k = h;
  p.seg_n = h;
  p.epi = kEpiStoreF32;
  p.fmt_bf16 = 1;
  p.out[0] = out;
  p.ldo = h;
  p.status = status;
  p.timeout_ns = kDefaultTimeoutNs;
  return launch_gemm(p, bn, st);
}

// ---------------------------------------------------------------- tensor-parallel baseline layer
// One tensor-parallel rank k of D holds head group k (Wq, Wk, Wv columns, Wo
// rows) and FFN block k (W1 columns, W2 rows) - the same shards as TSP - but
// ALL T tokens.  Its workspace: status section, scheduler counters, LN output
// [T, h] fp16, Q_k, K_k, V_k and A_k [T, h/D] fp16, H_k [T, F/D] fp16.
struct TpLayout {
  size_t status, counters, xn, q, k, v, a, hbuf, total;
};

TpLayout tp_layout(const Sizes& s) {
  TpLayout t;
  const size_t Th = static_cast<size_t>(s.T) * s.h, Ths = static_cast<size_t>(s.T) * s.hs;
  size_t o = 0;
  t.status = o; o += align_up(256);
  t.counters = o; o += align_up(256);
  t.xn = o; o += align_up(Th * 2);
  t.q = o; o += align_up(Ths * 2);
  t.k = o; o += align_up(Ths * 2);
  t.v = o; o += align_up(Ths * 2);
  t.a = o; o += align_up(Ths * 2);
  t.hbuf = o; o += align_up(static_cast<size_t>(s.T) * s.Fs * 2);
  t.total = o;
  return t;
}

// The whole sequence as one "rank" (D = 1: chunks 0 and 1 in natural order).
Sizes whole_sequence(const Sizes& s) {
  Sizes w = s;
  w.D = 1;
  w.c = s.T / 2;
  w.c_pad = (w.c + 127) / 128 * 128;
  w.L = s.T;
  w.hs = s.h;
  w.Fs = s.F;
  return w;
}

// ---------------------------------------------------------------- allocation-free K/V projection
// Scratch for tsp_kv_project_noalloc: a file-scope device array, so the call
// needs no device allocation.  Layout: status word (256 B), 768 B spare, then
// the LN1 output xn fp16 [L, h].  Every GPU that loads this library holds the
// array until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr size_t kNoAllocXnOffset = 1024;

// Device address of the array in the CUDA context current on this thread.
// The address belongs to a context: after cudaDeviceReset, or if the primary
// context is released and created again, the module is loaded anew and the
// array can move.  So the cache is per device AND keyed on the context's
// unique ID (cuCtxGetId; IDs are never reused within a process), and the
// address is looked up again whenever the current context is not the one it
// was found in.  In host code the array's name is only a host-side stand-in:
// the device address comes from cudaGetSymbolAddress, called with the device
// current (the first call on a device, or in a new context, does this lookup).
struct NoAllocEntry {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;
  bool keyed = false;
};
std::mutex g_noalloc_mu;
NoAllocEntry g_noalloc_cache[256];

// ID of the context current on this thread; false if none is current or the
// driver entry points are unavailable (then every call looks the address up).
bool current_ctx_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_cur = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_cur || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

int noalloc_scratch(void** out) {
  int dev = 0;
  TSP_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) return TSP_ERR_UNSUPPORTED;
  unsigned long long id = 0;
  const bool have_id = current_ctx_id(&id);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoAllocEntry& e = g_noalloc_cache[dev];
  if (have_id && e.keyed && e.addr && e.ctx_id == id) {
    *out = e.addr;
    return TSP_OK;
  }
  void* p = nullptr;
  TSP_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
  // the lookup makes the device's primary context current if none was
  unsigned long long id2 = 0;
  e.keyed = current_ctx_id(&id2);
  e.ctx_id = id2;
  e.addr = p;
  *out = p;
  return TSP_OK;
}

// The status section's two words -> the status a caller sees: a timeout
// first, then a failed debug-build index check, then a saturation; anything
// else in the status word is unknown.
int status_of_words(const int (&h)[2]) {
  if (h[0] == TSP_ERR_TIMEOUT) return TSP_ERR_TIMEOUT;
  if (h[0] != 0) return TSP_ERR_CUDA;
  if (h[1] & kFlagBoundsCheck) return TSP_ERR_BOUNDS;
  return (h[1] & kFlagFp16Saturated) ? TSP_ERR_SATURATED : TSP_OK;
}

}  // namespace

// ============================================================================
// C ABI
// ============================================================================
extern "C" {

const char* tsp_status_string(int status) {
  switch (status) {
    case TSP_OK: return "ok";
    case TSP_ERR_INVALID_ARG: return "invalid argument";
    case TSP_ERR_UNSUPPORTED: return "unsupported shape";
    case TSP_ERR_CUDA: return "CUDA error";
    case TSP_ERR_TIMEOUT: return "device wait timed out";
    case TSP_ERR_WORKSPACE: return "workspace too small";
    case TSP_ERR_SATURATED: return "fp16 conversion saturated";
    case TSP_ERR_BOUNDS: return "device index check failed";
    default: return "unknown status";
  }
}

const char* tsp_last_cuda_error(void) { return g_cuda_err; }

int tsp_check_dims(const tsp_dims* dims, int D) { return check_dims(dims, D); }

int tsp_zigzag_index(int64_t T, int D, int rank, int32_t* d_idx, cudaStream_t stream) {
  TSP_RANGE("tsp_zigzag_index");
  if (D < 1 || D > TSP_MAX_D || rank < 0 || rank >= D || T < 0 || T % (2 * D) != 0) return TSP_ERR_INVALID_ARG;
  if (T >= (int64_t(1) << 31)) return TSP_ERR_UNSUPPORTED;
  const int64_t c = T / (2 * D);
  if (c == 0) return TSP_OK;
  if (!d_idx) return TSP_ERR_INVALID_ARG;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((2 * c + threads - 1) / threads);
  zigzag_index_kernel<<<blocks, threads, 0, stream>>>(d_idx, c, D, rank);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

size_t tsp_shard_buffer_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  const size_t h = dims->h, F = dims->ffn;
  // a status section, then per shard: 4 attention matrices of h*h/D, 2 FFN
  // matrices of h*F/D
  return kAlign + static_cast<size_t>(D) * (4 * align_up(h * (h / D) * 2) + 2 * align_up(h * (F / D) * 2));
}

int tsp_pack_shards(const tsp_dims* dims, int D, const void* const w_full[6], void* d_buf, size_t buf_bytes,
                    tsp_weights* out, cudaStream_t stream) {
  TSP_RANGE("tsp_pack_shards");
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if (!w_full || !d_buf || !out) return TSP_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!w_full[i]) return TSP_ERR_INVALID_ARG;
  if (buf_bytes < tsp_shard_buffer_bytes(dims, D)) return TSP_ERR_WORKSPACE;
  const int h = dims->h, F = dims->ffn, hs = h / D, Fs = F / D;
  if (!aligned16(d_buf)) return TSP_ERR_INVALID_ARG;
  std::memset(out, 0, sizeof(*out));
  out->D = D;
  int* status = static_cast<int*>(d_buf);  // status section: status word, flags word
  TSP_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(int), stream));
  uint8_t* p = static_cast<uint8_t*>(d_buf) + kAlign;
  const dim3 blk(32, 8);
  auto pack = [&](const void* src, int64_t ld, int64_t row0, int64_t col0, int n_out, int n_in, const void** dst) -> int {
    *dst = p;
    const dim3 grid((n_in + 31) / 32, (n_out + 31) / 32);
    pack_transpose_kernel<<<grid, blk, 0, stream>>>(static_cast<const __nv_bfloat16*>(src), ld, row0, col0,
                                                    reinterpret_cast<__half*>(p), n_out, n_in, status);
    TSP_CUDA(cudaGetLastError());
    p += align_up(static_cast<size_t>(n_out) * n_in * 2);
    return TSP_OK;
  };
  for (int k = 0; k < D; ++k) {
    // column shards (head group / FFN block k of the output features): [n/D, in]
    if ((rc = pack(w_full[0], h, 0, int64_t(k) * hs, hs, h, &out->wq[k]))) return rc;
    if ((rc = pack(w_full[1], h, 0, int64_t(k) * hs, hs, h, &out->wk[k]))) return rc;
    if ((rc = pack(w_full[2], h, 0, int64_t(k) * hs, hs, h, &out->wv[k]))) return rc;
    // row shards (the same head group / FFN block on the input side): [h, in/D]
    if ((rc = pack(w_full[3], h, int64_t(k) * hs, 0, h, hs, &out->wo[k]))) return rc;
    if ((rc = pack(w_full[4], F, 0, int64_t(k) * Fs, Fs, h, &out->w1[k]))) return rc;
    if ((rc = pack(w_full[5], h, int64_t(k) * Fs, 0, h, Fs, &out->w2[k]))) return rc;
  }
  return TSP_OK;
}

size_t tsp_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return ws_layout(sizes_of(dims, D)).total;
}

int tsp_workspace_offsets(const tsp_dims* dims, int D, size_t off[TSP_N_WS_OFFSETS]) {
  if (!off) return TSP_ERR_INVALID_ARG;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  const WsLayout w = ws_layout(sizes_of(dims, D));
  off[0] = w.status; off[1] = w.xn; off[2] = w.q; off[3] = w.a;
  off[4] = w.y1; off[5] = w.hbuf; off[6] = w.counters; off[7] = w.total;
  off[8] = w.lse;
  return TSP_OK;
}

size_t tsp_attn_backward_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return abwd_layout(sizes_of(dims, D)).total;
}

int tsp_attn_backward(const tsp_dims* dims, int D, int rank, const void* q, const void* k_full, const void* v_full,
                      const void* o, const void* lse, const void* d_o, void* dq, void* dk_full, void* dv_full,
                      void* ws, size_t ws_bytes, cudaStream_t stream) {
  TSP_RANGE("tsp_attn_backward");
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if (rank < 0 || rank >= D) return TSP_ERR_INVALID_ARG;
  const Sizes s = sizes_of(dims, D);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  const AbwdLayout b = abwd_layout(s);
  if (ws_bytes < b.total) return TSP_ERR_WORKSPACE;
  if (s.L == 0) return TSP_OK;
  const void* ptrs[10] = {q, k_full, v_full, o, lse, d_o, dq, dk_full, dv_full, nullptr};
  for (int i = 0; i < 9; ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return TSP_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  return launch_attn_backward(s, rank, dims, static_cast<const __half*>(q), k_full, v_full,
                              static_cast<const __half*>(o), static_cast<const float*>(lse),
                              static_cast<const __half*>(d_o), static_cast<float*>(dq), static_cast<float*>(dk_full),
                              static_cast<float*>(dv_full), reinterpret_cast<float*>(base + b.delta),
                              reinterpret_cast<int*>(base + b.counters), reinterpret_cast<int*>(base + b.status),
                              stream);
}

int tsp_reset_device_status(void* ws, cudaStream_t stream) {
  if (!ws) return TSP_ERR_INVALID_ARG;
  TSP_CUDA(cudaMemsetAsync(ws, 0, 2 * sizeof(int), stream));
  return TSP_OK;
}

int tsp_get_device_status(const void* ws, cudaStream_t stream) {
  if (!ws) return TSP_ERR_INVALID_ARG;
  int h[2] = {0, 0};
  TSP_CUDA(cudaMemcpyAsync(h, ws, sizeof(h), cudaMemcpyDeviceToHost, stream));
  TSP_CUDA(cudaStreamSynchronize(stream));
  return status_of_words(h);
}

int tsp_kv_project(const tsp_dims* dims, const tsp_weights* w, int rank, const void* x_local, void* k_full,
                   void* v_full, void* ws, size_t ws_bytes, cudaStream_t stream) {
  TSP_RANGE("tsp_kv_project");
  Ctx c;
  int rc = make_ctx(c, dims, w, rank, ws, ws_bytes);
  if (rc) return rc;
  if (c.s.L == 0) return TSP_OK;
  if (!x_local || !k_full || !v_full || !aligned16(x_local) || !aligned16(k_full) || !aligned16(v_full))
    return TSP_ERR_INVALID_ARG;
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), c.xn, c.s.L, c.s.h, dims->ln_eps,
                                       stream);
  if (rc) return rc;
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(w->wk),
                               reinterpret_cast<const void* const*>(w->wv), nullptr};
  void* out[3] = {k_full, v_full, nullptr};
  const int remap[3] = {1, 1, 0};
  return launch_proj(c.s, rank, c.xn, fam, out, remap, 2, kEpiStoreF16, c.s.h, c.status, stream);
}

int tsp_kv_project_noalloc(const tsp_dims* dims, const tsp_weights* w, int rank, const void* x_local, void* k_full,
                           void* v_full, cudaStream_t stream) {
  TSP_RANGE("tsp_kv_project_noalloc");
  const int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if ((rc = check_weights(w, D))) return rc;
  if (rank < 0 || rank >= D) return TSP_ERR_INVALID_ARG;
  const Sizes sz = sizes_of(dims, D);
  if (sz.L == 0) return TSP_OK;
  if (!x_local || !k_full || !v_full || !aligned16(x_local) || !aligned16(k_full) || !aligned16(v_full))
    return TSP_ERR_INVALID_ARG;
  const size_t need = kNoAllocXnOffset + static_cast<size_t>(sz.L) * sz.h * 2;
  if (need > kNoAllocScratchBytes) {
    std::snprintf(g_cuda_err, sizeof(g_cuda_err),
                  "tsp_kv_project_noalloc: T/D * h * 2 + 1024 = %zu bytes exceeds the %zu-byte static scratch", need,
                  kNoAllocScratchBytes);
    return TSP_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if ((rc = noalloc_scratch(&scratch))) return rc;
  uint8_t* base = static_cast<uint8_t*>(scratch);
  int* status = reinterpret_cast<int*>(base);
  __half* xn = reinterpret_cast<__half*>(base + kNoAllocXnOffset);
  // the array keeps the previous call's contents: the status and flags words
  // start at zero
  TSP_CUDA(cudaMemsetAsync(status, 0, 2 * sizeof(int), stream));
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), xn, sz.L, sz.h, dims->ln_eps, stream);
  if (rc) return rc;
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(w->wk),
                               reinterpret_cast<const void* const*>(w->wv), nullptr};
  void* out[3] = {k_full, v_full, nullptr};
  const int remap[3] = {1, 1, 0};
  return launch_proj(sz, rank, xn, fam, out, remap, 2, kEpiStoreF16, sz.h, status, stream);
}

int tsp_kv_project_noalloc_status(cudaStream_t stream) {
  void* scratch = nullptr;
  int rc = noalloc_scratch(&scratch);
  if (rc) return rc;
  int h[2] = {0, 0};
  TSP_CUDA(cudaMemcpyAsync(h, scratch, sizeof(h), cudaMemcpyDeviceToHost, stream));
  TSP_CUDA(cudaStreamSynchronize(stream));
  return status_of_words(h);
}

int tsp_layer_forward(const tsp_dims* dims, const tsp_weights* w, int rank, const void* x_local, const void* k_full,
                      const void* v_full, void* y_local, int y_dtype, void* ws, size_t ws_bytes, cudaStream_t stream,
                      cudaEvent_t* step_events) {
  TSP_RANGE("tsp_layer_forward");
  Ctx c;
  int rc = make_ctx(c, dims, w, rank, ws, ws_bytes);
  if (rc) return rc;
  if (y_dtype != TSP_OUT_BF16 && y_dtype != TSP_OUT_F32) return TSP_ERR_INVALID_ARG;
  if (c.s.L == 0) return TSP_OK;
  if (!x_local || !k_full || !v_full || !y_local || !aligned16(x_local) || !aligned16(k_full) ||
      !aligned16(v_full) || !aligned16(y_local))
    return TSP_ERR_INVALID_ARG;
  if ((rc = record(step_events, 0, stream))) return rc;
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), c.xn, c.s.L, c.s.h, dims->ln_eps,
                                       stream);
  if (rc) return rc;
  if ((rc = record(step_events, 1, stream))) return rc;
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(w->wq), nullptr, nullptr};
  void* out[3] = {c.q, nullptr, nullptr};
  const int remap[3] = {0, 0, 0};
  rc = launch_proj(c.s, rank, c.xn, fam, out, remap, 1, kEpiStoreF16, c.s.h, c.status, stream);
  if (rc) return rc;
  if ((rc = record(step_events, 2, stream))) return rc;
  return layer_tail(c, dims, w, rank, x_local, k_full, v_full, y_local, y_dtype, stream, step_events);
}

int tsp_rank_step(const tsp_dims* dims, const tsp_weights* w, int rank, const void* x_local, void* k_full,
                  void* v_full, void* y_local, int y_dtype, void* ws, size_t ws_bytes, cudaStream_t stream,
                  cudaEvent_t* step_events) {
  TSP_RANGE("tsp_rank_step");
  Ctx c;
  int rc = make_ctx(c, dims, w, rank, ws, ws_bytes);
  if (rc) return rc;
  if (y_dtype != TSP_OUT_BF16 && y_dtype != TSP_OUT_F32) return TSP_ERR_INVALID_ARG;
  if (c.s.L == 0) return TSP_OK;
  if (!x_local || !k_full || !v_full || !y_local || !aligned16(x_local) || !aligned16(k_full) ||
      !aligned16(v_full) || !aligned16(y_local))
    return TSP_ERR_INVALID_ARG;
  if ((rc = record(step_events, 0, stream))) return rc;
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), c.xn, c.s.L, c.s.h, dims->ln_eps,
                                       stream);
  if (rc) return rc;
  if ((rc = record(step_events, 1, stream))) return rc;
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(w->wq),
                               reinterpret_cast<const void* const*>(w->wk),
                               reinterpret_cast<const void* const*>(w->wv)};
  void* out[3] = {c.q, k_full, v_full};
  const int remap[3] = {0, 1, 1};
  rc = launch_proj(c.s, rank, c.xn, fam, out, remap, 3, kEpiStoreF16, c.s.h, c.status, stream);
  if (rc) return rc;
  if ((rc = record(step_events, 2, stream))) return rc;
  return layer_tail(c, dims, w, rank, x_local, k_full, v_full, y_local, y_dtype, stream, step_events);
}

int tsp_rank_step_host(const tsp_dims* dims, const tsp_weights* w, int rank, const void* h_x_local,
                       void* d_x_staging, void* k_full, void* v_full, void* d_y_staging, void* h_y_local, int y_dtype,
                       void* ws, size_t ws_bytes, cudaStream_t stream, cudaEvent_t compute_after,
                       cudaEvent_t compute_done) {
  TSP_RANGE("tsp_rank_step_host");
  Ctx c;
  int rc = make_ctx(c, dims, w, rank, ws, ws_bytes);
  if (rc) return rc;
  // every argument tsp_rank_step checks, before anything is enqueued
  if (y_dtype != TSP_OUT_BF16 && y_dtype != TSP_OUT_F32) return TSP_ERR_INVALID_ARG;
  if (c.s.L == 0) return TSP_OK;
  if (!h_x_local || !d_x_staging || !d_y_staging || !h_y_local || !k_full || !v_full) return TSP_ERR_INVALID_ARG;
  if (!aligned16(d_x_staging) || !aligned16(d_y_staging) || !aligned16(k_full) || !aligned16(v_full))
    return TSP_ERR_INVALID_ARG;
  const size_t xb = static_cast<size_t>(c.s.L) * c.s.h * 2;
  const size_t yb = static_cast<size_t>(c.s.L) * c.s.h * (y_dtype == TSP_OUT_F32 ? 4 : 2);
  TSP_CUDA(cudaMemcpyAsync(d_x_staging, h_x_local, xb, cudaMemcpyHostToDevice, stream));
  if (compute_after) TSP_CUDA(cudaStreamWaitEvent(stream, compute_after, 0));
  rc = tsp_rank_step(dims, w, rank, d_x_staging, k_full, v_full, d_y_staging, y_dtype, ws, ws_bytes, stream, nullptr);
  if (rc) return rc;
  if (compute_done) TSP_CUDA(cudaEventRecord(compute_done, stream));
  TSP_CUDA(cudaMemcpyAsync(h_y_local, d_y_staging, yb, cudaMemcpyDeviceToHost, stream));
  return TSP_OK;
}

size_t tsp_mlp_backward_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return bwd_layout(sizes_of(dims, D)).total;
}

int tsp_mlp_backward(const tsp_dims* dims, const tsp_weights* w, const void* w1_full, const void* w2_full,
                     const void* y1, const void* dy, void* dy1, void* dw1, void* dw2, void* bws, size_t bws_bytes,
                     cudaStream_t stream, cudaEvent_t* ev) {
  TSP_RANGE("tsp_mlp_backward");
  const int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  rc = check_weights(w, D);
  if (rc) return rc;
  const Sizes s = sizes_of(dims, D);
  // with no tokens only the weight gradients (zeros) are written
  const void* ptrs[7] = {w1_full, w2_full, dw1, dw2, y1, dy, dy1};
  for (int i = 0; i < (s.L == 0 ? 4 : 7); ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return TSP_ERR_INVALID_ARG;
  if (!bws || (reinterpret_cast<uintptr_t>(bws) & 255)) return TSP_ERR_INVALID_ARG;
  if ((rc = check_backward_shape(s))) return rc;
  const BwdLayout b = bwd_layout(s);
  if (bws_bytes < b.total) return TSP_ERR_WORKSPACE;
  return mlp_backward_core(s, dims, w, w1_full, w2_full, static_cast<const float*>(y1),
                           static_cast<const __nv_bfloat16*>(dy), static_cast<float*>(dy1), nullptr,
                           static_cast<float*>(dw1), static_cast<float*>(dw2), static_cast<uint8_t*>(bws), b, stream,
                           ev);
}

size_t tsp_layer_backward_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return lbwd_layout(sizes_of(dims, D)).total;
}

size_t tsp_kv_backward_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return kvbwd_layout(sizes_of(dims, D)).total;
}

int tsp_layer_backward(const tsp_dims* dims, const tsp_weights* w, const void* const w_full[6], int rank,
                       const void* x_local, const void* fwd_ws, size_t fwd_ws_bytes, const void* k_full,
                       const void* v_full, const void* dy, void* dx, void* dwq, void* dwo, void* dw1, void* dw2,
                       void* dk_full, void* dv_full, void* bws, size_t bws_bytes, cudaStream_t stream,
                       cudaEvent_t* ev) {
  TSP_RANGE("tsp_layer_backward");
  const int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if ((rc = check_weights(w, D))) return rc;
  if (rank < 0 || rank >= D || !w_full) return TSP_ERR_INVALID_ARG;
  const Sizes s = sizes_of(dims, D);
  for (int i = 0; i < 6; ++i)
    if (!w_full[i] || !aligned16(w_full[i])) return TSP_ERR_INVALID_ARG;
  const void* ptrs[11] = {dwq, dwo, dw1, dw2, x_local, fwd_ws, k_full, v_full, dy, dx, dk_full};
  for (int i = 0; i < (s.L == 0 ? 4 : 11); ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return TSP_ERR_INVALID_ARG;
  if (s.L > 0 && (!dv_full || !aligned16(dv_full))) return TSP_ERR_INVALID_ARG;
  if (!bws || (reinterpret_cast<uintptr_t>(bws) & 255)) return TSP_ERR_INVALID_ARG;
  if ((rc = check_backward_shape(s))) return rc;
  const LayerBwdLayout lb = lbwd_layout(s);
  if (bws_bytes < lb.total) return TSP_ERR_WORKSPACE;
  const WsLayout fl = ws_layout(s);
  if (s.L > 0 && fwd_ws_bytes < fl.total) return TSP_ERR_WORKSPACE;
  const size_t hh = static_cast<size_t>(s.h) * s.h * 4;
  if ((rc = record(ev, 0, stream))) return rc;
  if (s.L == 0) {  // no tokens: zero weight gradients
    TSP_CUDA(cudaMemsetAsync(dwq, 0, hh, stream));
    TSP_CUDA(cudaMemsetAsync(dwo, 0, hh, stream));
    TSP_CUDA(cudaMemsetAsync(dw1, 0, static_cast<size_t>(s.h) * s.F * 4, stream));
    TSP_CUDA(cudaMemsetAsync(dw2, 0, static_cast<size_t>(s.F) * s.h * 4, stream));
    for (int i = 1; i < TSP_N_STEP_EVENTS; ++i)
      if ((rc = record(ev, i, stream))) return rc;
    return TSP_OK;
  }
  uint8_t* base = static_cast<uint8_t*>(bws);
  int* status = reinterpret_cast<int*>(base + lb.mlp.status);
  const uint8_t* fws = static_cast<const uint8_t*>(fwd_ws);
  const __half* q = reinterpret_cast<const __half*>(fws + fl.q);
  const __half* a = reinterpret_cast<const __half*>(fws + fl.a);
  const float* y1 = reinterpret_cast<const float*>(fws + fl.y1);
  const float* lse = reinterpret_cast<const float*>(fws + fl.lse);
  float* dy1 = reinterpret_cast<float*>(base + lb.dy1);
  __nv_bfloat16* dy1b = reinterpret_cast<__nv_bfloat16*>(base + lb.dy1b);
  __nv_bfloat16* dy1t = reinterpret_cast<__nv_bfloat16*>(base + lb.dy1t);
  __nv_bfloat16* at = reinterpret_cast<__nv_bfloat16*>(base + lb.at);
  __half* d_o = reinterpret_cast<__half*>(base + lb.d_o);
  float* dq = reinterpret_cast<float*>(base + lb.dq);
  __nv_bfloat16* dqb = reinterpret_cast<__nv_bfloat16*>(base + lb.dqb);
  __nv_bfloat16* dqt = reinterpret_cast<__nv_bfloat16*>(base + lb.dqt);
  __half* xn1 = reinterpret_cast<__half*>(base + lb.xn1);
  __nv_bfloat16* xn1t = reinterpret_cast<__nv_bfloat16*>(base + lb.xn1t);
  float* dxn1 = reinterpret_cast<float*>(base + lb.dxn1);
  const int L = static_cast<int>(s.L);
  // MLP half: dY1 (and its bf16 copy), dW1, dW2
  rc = mlp_backward_core(s, dims, w, w_full[4], w_full[5], y1, static_cast<const __nv_bfloat16*>(dy), dy1, dy1b,
                         static_cast<float*>(dw1), static_cast<float*>(dw2), base, lb.mlp, stream, nullptr);
  if (rc) return rc;
  if ((rc = record(ev, 1, stream))) return rc;
  // dA = dY1 Wo^T (Wo [h_in, h_out] row-major is K-major over h_out), fp16 for
  // the attention backward's tensor cores
  rc = launch_plain(dy1b, L, s.h, s.h, w_full[3], s.h, s.h, true, kEpiStoreF16, d_o, s.h, nullptr, status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 2, stream))) return rc;
  // dWo = A^T dY1: both operands token-major
  if ((rc = launch_transpose<__half>(a, s.L, s.h, at, stream))) return rc;
  if ((rc = launch_transpose<float>(dy1, s.L, s.h, dy1t, stream))) return rc;
  rc = launch_plain(at, s.h, L, L, dy1t, s.h, L, true, kEpiStoreF32, dwo, s.h, nullptr, status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 3, stream))) return rc;
  // the attention: dQ, and this rank's dK, dV for all keys
  rc = launch_attn_backward(s, rank, dims, q, k_full, v_full, a, lse, d_o, dq, static_cast<float*>(dk_full),
                            static_cast<float*>(dv_full), reinterpret_cast<float*>(base + lb.delta),
                            reinterpret_cast<int*>(base + lb.counters), status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 4, stream))) return rc;
  // bf16 copies of dQ (row-major and token-major), LN1(x) recomputed
  if ((rc = launch_convert_bf16(dq, dqb, static_cast<int64_t>(s.L) * s.h, stream))) return rc;
  if ((rc = launch_transpose<float>(dq, s.L, s.h, dqt, stream))) return rc;
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), xn1, s.L, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  if ((rc = launch_transpose<__half>(xn1, s.L, s.h, xn1t, stream))) return rc;
  if ((rc = record(ev, 5, stream))) return rc;
  // dWq = LN1(X)^T dQ
  rc = launch_plain(xn1t, s.h, L, L, dqt, s.h, L, true, kEpiStoreF32, dwq, s.h, nullptr, status, stream);
  if (rc) return rc;
  if ((rc = record(ev, 6, stream))) return rc;
  // dX = dY1 + LN1'(X)^T (dQ Wq^T)   (Wq [h_in, h_out] is K-major over h_out)
  rc = launch_plain(dqb, L, s.h, s.h, w_full[0], s.h, s.h, true, kEpiStoreF32, dxn1, s.h, nullptr, status, stream);
  if (rc) return rc;
  rc = launch_ln_backward<__nv_bfloat16, float>(static_cast<const __nv_bfloat16*>(x_local), dxn1, dy1,
                                                static_cast<float*>(dx), nullptr, s.L, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  return record(ev, 7, stream);
}

int tsp_kv_backward(const tsp_dims* dims, int D, const void* const w_full[6], int rank, const void* x_local,
                    const void* dk_full, const void* dv_full, void* dx, void* dwk, void* dwv, void* kws,
                    size_t kws_bytes, cudaStream_t stream) {
  TSP_RANGE("tsp_kv_backward");
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if (rank < 0 || rank >= D || !w_full) return TSP_ERR_INVALID_ARG;
  const Sizes s = sizes_of(dims, D);
  if (!w_full[1] || !w_full[2] || !aligned16(w_full[1]) || !aligned16(w_full[2])) return TSP_ERR_INVALID_ARG;
  const void* ptrs[7] = {dwk, dwv, x_local, dk_full, dv_full, dx, nullptr};
  for (int i = 0; i < (s.L == 0 ? 2 : 6); ++i)
    if (!ptrs[i] || !aligned16(ptrs[i])) return TSP_ERR_INVALID_ARG;
  if (!kws || (reinterpret_cast<uintptr_t>(kws) & 255)) return TSP_ERR_INVALID_ARG;
  if ((rc = check_backward_shape(s))) return rc;
  const KvBwdLayout kb = kvbwd_layout(s);
  if (kws_bytes < kb.total) return TSP_ERR_WORKSPACE;
  const size_t hh = static_cast<size_t>(s.h) * s.h * 4;
  if (s.L == 0) {
    TSP_CUDA(cudaMemsetAsync(dwk, 0, hh, stream));
    TSP_CUDA(cudaMemsetAsync(dwv, 0, hh, stream));
    return TSP_OK;
  }
  uint8_t* base = static_cast<uint8_t*>(kws);
  int* status = reinterpret_cast<int*>(base + kb.status);
  __half* xn1 = reinterpret_cast<__half*>(base + kb.xn1);
  __nv_bfloat16* xn1t = reinterpret_cast<__nv_bfloat16*>(base + kb.xn1t);
  __nv_bfloat16* kv = reinterpret_cast<__nv_bfloat16*>(base + kb.kv);
  __nv_bfloat16* kvt = reinterpret_cast<__nv_bfloat16*>(base + kb.kvt);
  float* dxn = reinterpret_cast<float*>(base + kb.dxn);
  const int L = static_cast<int>(s.L);
  // the rank's rows of the summed dK, dV: [dK | dV] bf16 [L, 2h], and
  // token-major [2h, L]
  {
    const int64_t threads = s.L * (2 * s.h / 8);
    gather_kv_grad_kernel<<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(
        static_cast<const float*>(dk_full), static_cast<const float*>(dv_full), kv, s.L, s.h, s.c,
        static_cast<int64_t>(rank) * s.c, static_cast<int64_t>(2 * s.D - 1 - rank) * s.c - s.c);
    TSP_CUDA(cudaGetLastError());
  }
  if ((rc = launch_transpose<__nv_bfloat16>(kv, s.L, 2 * s.h, kvt, stream))) return rc;
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x_local), xn1, s.L, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  if ((rc = launch_transpose<__half>(xn1, s.L, s.h, xn1t, stream))) return rc;
  // dWk = LN1(X)^T dK, dWv = LN1(X)^T dV
  rc = launch_plain(xn1t, s.h, L, L, kvt, s.h, L, true, kEpiStoreF32, dwk, s.h, nullptr, status, stream);
  if (rc) return rc;
  rc = launch_plain(xn1t, s.h, L, L, kvt + static_cast<size_t>(s.h) * s.L, s.h, L, true, kEpiStoreF32, dwv, s.h,
                    nullptr, status, stream);
  if (rc) return rc;
  // dXn = dK Wk^T + dV Wv^T: one K-split product over [dK | dV] with the two
  // weights as its two K blocks; then dX += LN1'(X)^T dXn
  rc = launch_kv_grad_input(kv, L, s.h, w_full[1], w_full[2], dxn, status, stream);
  if (rc) return rc;
  return launch_ln_backward<__nv_bfloat16, float>(static_cast<const __nv_bfloat16*>(x_local), dxn,
                                                  static_cast<const float*>(dx), static_cast<float*>(dx), nullptr,
                                                  s.L, s.h, dims->ln_eps, stream);
}

size_t tsp_tp_workspace_bytes(const tsp_dims* dims, int D) {
  if (check_dims(dims, D) != TSP_OK) return 0;
  return tp_layout(sizes_of(dims, D)).total;
}

int tsp_tp_attention_partial(const tsp_dims* dims, const tsp_weights* w, int k, const void* x, void* part, void* ws,
                             size_t ws_bytes, cudaStream_t stream) {
  TSP_RANGE("tsp_tp_attention_partial");
  const int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if ((rc = check_weights(w, D))) return rc;
  if (k < 0 || k >= D) return TSP_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  const Sizes s = sizes_of(dims, D);
  const TpLayout t = tp_layout(s);
  if (ws_bytes < t.total) return TSP_ERR_WORKSPACE;
  if (s.T == 0) return TSP_OK;
  if (!x || !part || !aligned16(x) || !aligned16(part)) return TSP_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base + t.status);
  __half* xn = reinterpret_cast<__half*>(base + t.xn);
  __half* q = reinterpret_cast<__half*>(base + t.q);
  __half* kk = reinterpret_cast<__half*>(base + t.k);
  __half* v = reinterpret_cast<__half*>(base + t.v);
  __half* a = reinterpret_cast<__half*>(base + t.a);
  const Sizes full = whole_sequence(s);
  // LN1 of every token (each tensor-parallel rank computes it)
  rc = launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), xn, s.T, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  // Q_k, K_k, V_k = LN1(X) [Wq_k | Wk_k | Wv_k]: the column-parallel product
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(&w->wq[k]),
                               reinterpret_cast<const void* const*>(&w->wk[k]),
                               reinterpret_cast<const void* const*>(&w->wv[k])};
  void* out[3] = {q, kk, v};
  const int noremap[3] = {0, 0, 0};
  rc = launch_proj(full, 0, xn, fam, out, noremap, 3, kEpiStoreF16, s.hs, status, stream);
  if (rc) return rc;
  // causal attention of head group k over the whole sequence
  tsp_dims dk = *dims;
  dk.h = s.hs;
  dk.n_heads = s.H / D;
  Sizes sa = full;
  sa.h = s.hs;
  sa.H = s.H / D;
  rc = launch_attention(sa, 0, &dk, q, kk, v, a, nullptr, reinterpret_cast<int*>(base + t.counters), status, stream);
  if (rc) return rc;
  // the row-parallel product A_k Wo_k^T: this rank's partial of the sum the
  // all-reduce forms
  return launch_plain(a, static_cast<int>(s.T), s.hs, s.hs, w->wo[k], s.h, s.hs, false, kEpiStoreF32, part, s.h,
                      nullptr, status, stream);
}

int tsp_tp_mlp_partial(const tsp_dims* dims, const tsp_weights* w, int k, const void* y1, void* part, void* ws,
                       size_t ws_bytes, cudaStream_t stream) {
  TSP_RANGE("tsp_tp_mlp_partial");
  const int D = w ? w->D : 0;
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if ((rc = check_weights(w, D))) return rc;
  if (k < 0 || k >= D) return TSP_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  const Sizes s = sizes_of(dims, D);
  const TpLayout t = tp_layout(s);
  if (ws_bytes < t.total) return TSP_ERR_WORKSPACE;
  if (s.T == 0) return TSP_OK;
  if (!y1 || !part || !aligned16(y1) || !aligned16(part)) return TSP_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base + t.status);
  __half* xn = reinterpret_cast<__half*>(base + t.xn);
  __half* hb = reinterpret_cast<__half*>(base + t.hbuf);
  const Sizes full = whole_sequence(s);
  rc = launch_layernorm<float>(static_cast<const float*>(y1), xn, s.T, s.h, dims->ln_eps, stream);
  if (rc) return rc;
  // H_k = GELU(LN2(Y1) W1_k) (column-parallel), then H_k W2_k^T (row-parallel)
  const void* const* fam[3] = {reinterpret_cast<const void* const*>(&w->w1[k]), nullptr, nullptr};
  void* out[3] = {hb, nullptr, nullptr};
  const int noremap[3] = {0, 0, 0};
  rc = launch_proj(full, 0, xn, fam, out, noremap, 1, kEpiGeluF16, s.Fs, status, stream);
  if (rc) return rc;
  return launch_plain(hb, static_cast<int>(s.T), s.Fs, s.Fs, w->w2[k], s.h, s.Fs, false, kEpiStoreF32, part, s.h,
                      nullptr, status, stream);
}

int tsp_tp_all_reduce(const tsp_dims* dims, int n_parts, const void* const parts[], const void* resid, int resid_f32,
                      void* out, int out_dtype, cudaStream_t stream) {
  TSP_RANGE("tsp_tp_all_reduce");
  if (!dims || n_parts < 1 || n_parts > TSP_MAX_D || !parts) return TSP_ERR_INVALID_ARG;
  if (dims->T < 0 || dims->h <= 0 || dims->h % 4) return TSP_ERR_INVALID_ARG;
  if (out_dtype != TSP_OUT_BF16 && out_dtype != TSP_OUT_F32) return TSP_ERR_INVALID_ARG;
  const int64_t n = dims->T * dims->h;
  if (n == 0) return TSP_OK;
  PartList pl = {};
  for (int i = 0; i < n_parts; ++i) {
    if (!parts[i] || !aligned16(parts[i])) return TSP_ERR_INVALID_ARG;
    pl.p[i] = static_cast<const float*>(parts[i]);
  }
  if (!resid || !out || !aligned16(resid) || !aligned16(out)) return TSP_ERR_INVALID_ARG;
  const unsigned blocks = static_cast<unsigned>((n / 4 + 255) / 256);
  const bool of = out_dtype == TSP_OUT_F32;
  if (resid_f32) {
    if (of) sum_partials_kernel<float, true><<<blocks, 256, 0, stream>>>(pl, n_parts, static_cast<const float*>(resid), out, n);
    else sum_partials_kernel<float, false><<<blocks, 256, 0, stream>>>(pl, n_parts, static_cast<const float*>(resid), out, n);
  } else {
    const __nv_bfloat16* r = static_cast<const __nv_bfloat16*>(resid);
    if (of) sum_partials_kernel<__nv_bfloat16, true><<<blocks, 256, 0, stream>>>(pl, n_parts, r, out, n);
    else sum_partials_kernel<__nv_bfloat16, false><<<blocks, 256, 0, stream>>>(pl, n_parts, r, out, n);
  }
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

// ---------------------------------------------------------------- per-shard steps
namespace {

// Sizes of one head group (shard) of the attention: h/D columns, H/D heads.
Sizes head_group(const Sizes& s) {
  Sizes g = s;
  g.h = s.hs;
  g.H = s.H / s.D;
  return g;
}

int shard_args(const tsp_dims* dims, int D, int rank, Sizes* s) {
  int rc = check_dims(dims, D);
  if (rc) return rc;
  if (rank < 0 || rank >= D) return TSP_ERR_INVALID_ARG;
  *s = sizes_of(dims, D);
  return TSP_OK;
}

bool ok16(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p || !aligned16(p)) return false;
  return true;
}

int* status_of(void* ws) { return static_cast<int*>(ws); }

}  // namespace

size_t tsp_shard_workspace_bytes(void) { return 2 * kAlign; }

int tsp_layernorm(int64_t rows, int h, float eps, const void* x, int x_f32, void* y, cudaStream_t stream) {
  TSP_RANGE("tsp_layernorm");
  if (rows < 0 || h <= 0 || h % 8 || h > 8192 || !(eps >= 0.f)) return TSP_ERR_INVALID_ARG;
  if (rows == 0) return TSP_OK;
  if (!ok16({x, y})) return TSP_ERR_INVALID_ARG;
  if (x_f32) return launch_layernorm<float>(static_cast<const float*>(x), static_cast<__half*>(y), rows, h, eps, stream);
  return launch_layernorm<__nv_bfloat16>(static_cast<const __nv_bfloat16*>(x), static_cast<__half*>(y), rows, h, eps,
                                         stream);
}

int tsp_shard_qkv(const tsp_dims* dims, int D, int rank, const void* wq_k, const void* wk_k, const void* wv_k,
                  const void* xn1, void* q_k, void* k_k, void* v_k, void* ws, cudaStream_t stream) {
  TSP_RANGE("tsp_shard_qkv");
  Sizes s;
  int rc = shard_args(dims, D, rank, &s);
  if (rc) return rc;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  if (s.L == 0) return TSP_OK;
  if (!ok16({wq_k, wk_k, wv_k, xn1, q_k, k_k, v_k})) return TSP_ERR_INVALID_ARG;
  const void* wq[1] = {wq_k};
  const void* wk[1] = {wk_k};
  const void* wv[1] = {wv_k};
  const void* const* fam[3] = {wq, wk, wv};
  void* out[3] = {q_k, k_k, v_k};
  const int remap[3] = {0, 1, 1};  // K, V rows to their global positions
  Sizes one = s;
  one.D = 1;  // one shard per segment; the zigzag rows still follow (rank, D)
  return launch_proj_zz(s, one, rank, static_cast<const __half*>(xn1), fam, out, remap, 3, kEpiStoreF16, s.hs,
                        status_of(ws), stream);
}

int tsp_shard_attention(const tsp_dims* dims, int D, int rank, const void* q_k, const void* k_k, const void* v_k,
                        void* a_k, void* ws, cudaStream_t stream) {
  TSP_RANGE("tsp_shard_attention");
  Sizes s;
  int rc = shard_args(dims, D, rank, &s);
  if (rc) return rc;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  if (s.L == 0) return TSP_OK;
  if (!ok16({q_k, k_k, v_k, a_k})) return TSP_ERR_INVALID_ARG;
  tsp_dims dg = *dims;
  dg.h = s.hs;
  dg.n_heads = s.H / D;
  uint8_t* base = static_cast<uint8_t*>(ws);
  return launch_attention(head_group(s), rank, &dg, static_cast<const __half*>(q_k), k_k, v_k,
                          static_cast<__half*>(a_k), nullptr, reinterpret_cast<int*>(base + kAlign),
                          status_of(ws), stream);
}

int tsp_shard_ffn_up(const tsp_dims* dims, int D, const void* w1_k, const void* xn2, void* h_k, void* ws,
                     cudaStream_t stream) {
  TSP_RANGE("tsp_shard_ffn_up");
  Sizes s;
  int rc = shard_args(dims, D, 0, &s);
  if (rc) return rc;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  if (s.L == 0) return TSP_OK;
  if (!ok16({w1_k, xn2, h_k})) return TSP_ERR_INVALID_ARG;
  const void* w1[1] = {w1_k};
  const void* const* fam[3] = {w1, nullptr, nullptr};
  void* out[3] = {h_k, nullptr, nullptr};
  const int noremap[3] = {0, 0, 0};
  Sizes one = s;
  one.D = 1;
  return launch_proj_zz(s, one, 0, static_cast<const __half*>(xn2), fam, out, noremap, 1, kEpiGeluF16, s.Fs,
                        status_of(ws), stream);
}

int tsp_shard_accumulate(const tsp_dims* dims, int D, const void* act, int k_dim, const void* w_k, void* y,
                         void* ws, cudaStream_t stream) {
  TSP_RANGE("tsp_shard_accumulate");
  Sizes s;
  int rc = shard_args(dims, D, 0, &s);
  if (rc) return rc;
  if (k_dim != s.hs && k_dim != s.Fs) return TSP_ERR_INVALID_ARG;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255)) return TSP_ERR_INVALID_ARG;
  if (s.L == 0) return TSP_OK;
  if (!ok16({act, w_k, y})) return TSP_ERR_INVALID_ARG;
  // y += act [L, k_dim] w_k^T (w_k K-major [h, k_dim]); the residual epilogue
  // reads each value of y before it writes it
  const void* fam[1] = {w_k};
  Sizes one = s;
  one.D = 1;
  return launch_ksplit(one, 0, static_cast<const __half*>(act), k_dim, fam, y, 1, y, 1, status_of(ws), stream);
}

int tsp_selftest_wait_timeout(void* ws, uint64_t timeout_ns, cudaStream_t stream) {
  if (timeout_ns == 0 || timeout_ns > 2000000000ull) return TSP_ERR_INVALID_ARG;
  if (!ws) {  // the status word of tsp_kv_project_noalloc's static scratch
    int rc = noalloc_scratch(&ws);
    if (rc) return rc;
  }
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<int*>(ws), timeout_ns);
  TSP_CUDA(cudaGetLastError());
  return TSP_OK;
}

}  // extern "C"
