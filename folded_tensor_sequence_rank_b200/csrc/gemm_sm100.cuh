// gemm_sm100.cuh - persistent tcgen05 GEMM C = A * B^T for the TSP shard loops.
//
// A [M, K] K-major (one tensor map), B given as a list of per-shard K-major
// tensor maps, both fp16 or both bf16 (fmt_bf16); fp32 accumulation in
// tensor memory.  Two ways the shard list is walked, both without any
// reduction kernel:
//   N-split (Q/K/V and W1 shards: each shard owns a block of output columns):
//     output column block n belongs to map n / shard_n.
//   K-split (Wo and W2 shards: each shard owns a block of the reduction dim):
//     k-block kb reads map (kb*64) / shard_k, so one TMEM accumulator sums the
//     contributions of all D shards - the "no all-reduce" MLP sum of the
//     TSP news item (zubnet.ai, paragraphs 2 and 4) done inside the K loop.
//
// Roles (192 threads, one CTA per SM, persistent over output tiles):
//   warp 0     TMA producer: A and B tiles into a STAGES-deep shared ring
//   warp 1     TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-5  epilogue: tcgen05.ld the 128 x BN fp32 accumulator (thread =
//              row), apply store / GELU / residual / GELU', write to global
//              memory (fp16 operands for the next matmul, the fp32 / bf16
//              residual stream, bf16 gradients, fp32 weight gradients).
// Two TMEM accumulators let the epilogue of tile i overlap the K loop of
// tile i+1.
#pragma once
#include "ptx.cuh"

namespace tsp {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmThreads = 192;
constexpr int kGemmMaxMaps = 48;  // 3 segments x 16 shards
constexpr int kGemmGroupM = 16;   // M tiles per raster group (L2 reuse of A)

// Epilogues.  kEpiStoreF16 / kEpiGeluF16 write fp16 operands for the next
// matmul, saturating at +-65504 and
// setting kFlagFp16Saturated in the flags word after `status` when a value
// was out of range; kEpiResidual adds the
// residual stream; kEpiGeluBwd writes the bf16 gradient acc * GELU'(U) with U
// (fp16, [M, ldo]) at `resid`; kEpiStoreF32 writes acc as fp32.
// kEpiStoreF16 and kEpiGeluBwd can also write the tile transposed, as bf16,
// to out_t [N, ld_t] (row n, column m): kEpiStoreF16 writes GELU of the
// fp16-rounded value there, kEpiGeluBwd the gradient itself.  A warp holds 32
// consecutive rows; it transposes each 32 x 32 chunk through its own slice of
// shared memory, so every lane writes one 64-byte output row segment.  The
// transposed store needs every lane of the warp (M a multiple of 128).
enum GemmEpi : int { kEpiStoreF16 = 0, kEpiGeluF16 = 1, kEpiResidual = 2, kEpiGeluBwd = 3, kEpiStoreF32 = 4 };

struct __align__(64) GemmParams {
  CUtensorMap map_a;
  CUtensorMap map_b[kGemmMaxMaps];
  CUtensorMap map_out;  // pair kernel, kEpiResidual with tma_out: the output as a store destination
  int tma_out;
  int M, N, K;
  int ksplit;     // 0: N-split, 1: K-split
  int shard_n;    // N-split: output columns per B map
  int shard_k;    // K-split: reduction length per B map
  int seg_n;      // N-split: output columns per output segment
  int epi;        // GemmEpi
  int fmt_bf16;   // operands: 0 fp16, 1 bf16
  void* out_t;    // optional transposed bf16 copy [N, ld_t] (see above)
  int64_t ld_t;
  void* out[3];   // per segment (N-split, fp16) or out[0] (K-split, fp32 / bf16)
  int remap[3];   // per segment: 1 = write local row m at its global zigzag row
  int64_t ldo;    // output row stride, elements
  const void* resid;  // kEpiResidual: residual [M, N] (row stride ldo)
  int resid_f32;      // residual dtype: 1 fp32, 0 bf16
  int out_f32;        // kEpiResidual: output fp32 (1) or bf16 (0)
  int c;              // zigzag: local rows [0,c) -> off0 + m, [c, 2c) -> off1 + m
  int64_t off0, off1;
  int64_t remap_rows;  // rows of a remapped (global-row) output: index checks of the debug build
  int* status;        // status word; status[1] is the flags word
  uint64_t timeout_ns;
};

// Per epilogue warp: 16 words x 32 rows, row stride 36 words (16-byte
// aligned, and the 128-bit reads of one transposed row spread over banks).
constexpr int kStageStride = 36;
constexpr int kStageWords = 16 * kStageStride;
constexpr int kStageBytes = 4 * kStageWords * 4;

template <int BN>
struct GemmShape {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStages = (BN == 256) ? 4 : (BN == 128 ? 6 : 8);
  static constexpr int kTmemCols = 2 * BN;  // two accumulators
  static constexpr int kBarBytes = 256;
  static constexpr int kSmemBytes = kStages * (kABytes + kBBytes) + kBarBytes + kStageBytes + 1024;
};

__device__ __forceinline__ void gemm_tile_coords(int tile, int num_m, int num_n, int& mb, int& nb) {
  const int per_group = kGemmGroupM * num_n;
  const int group = tile / per_group;
  const int first_m = group * kGemmGroupM;
  const int gm = min(kGemmGroupM, num_m - first_m);
  const int local = tile - group * per_group;
  mb = first_m + local % gm;
  nb = local / gm;
}

// GELU, tanh form, through the identity 0.5 (1 + tanh(u)) = 1 / (1 + e^(-2u)):
//   GELU(x) = x / (1 + 2^(-2 u log2(e))),  u = sqrt(2/pi) (x + 0.044715 x^3).
// ex2.approx has ~2^-22 relative error and the fast division (__fdividef) at
// most 2 ulps, so the result is accurate to a few fp32 ulps before its 16-bit
// rounding.  An IEEE-rounded division cost the W1 GEMM 8% of its time.  The
// fast division's limits are harmless here: a denominator beyond 2^126 (x <
// about -44) gives 0, GELU's limit; an infinite x, for which it would give
// NaN, cannot come out of a GEMM of finite fp16 operands.
__device__ __forceinline__ float gelu_tanh_f(float x) {
  const float k = -2.0f * 0.7978845608028654f * 1.4426950408889634f;  // -2 sqrt(2/pi) log2(e)
  const float u = fmaf(0.044715f * x, x * x, x);
  return __fdividef(x, 1.0f + ex2_approx(k * u));
}

// d/dx GELU (tanh form).  With p = 1 / (1 + e^(-2u)) = 0.5 (1 + tanh(u)),
// 1 - tanh(u)^2 = 4 p (1 - p), so
//   GELU'(x) = p + 2 x p (1 - p) sqrt(2/pi) (1 + 3 * 0.044715 x^2).
__device__ __forceinline__ float gelu_tanh_grad_f(float x) {
  const float s = 0.7978845608028654f;
  const float k = -2.0f * 0.7978845608028654f * 1.4426950408889634f;  // -2 sqrt(2/pi) log2(e)
  const float x2 = x * x;
  const float u = fmaf(0.044715f * x, x2, x);
  const float pr = __fdividef(1.0f, 1.0f + ex2_approx(k * u));  // as in gelu_tanh_f
  return fmaf(2.0f * x * pr * (1.0f - pr) * s, fmaf(3.0f * 0.044715f, x2, 1.0f), pr);
}

// Bounded wait that ignores the abort flag: used only to drain copies and
// MMAs this thread itself started, before the CTA exits.
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t a = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(a, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) break;
  }
}

// Writes the 32 x 32 bf16 chunk whose row m (this lane) holds w[k] =
// columns (n + 2k, n + 2k + 1) as rows n .. n+31 of out_t: each lane packs
// its words into `stage` (word k of row `lane` at k * kStageStride + lane),
// then reads back the column pair of output row n + lane with 128-bit loads
// and joins rows 2i, 2i+1 with a byte permute.
__device__ __forceinline__ void store_transposed_bf16(const GemmParams& p, uint32_t* stage, int m, int n,
                                                      const uint32_t (&w)[16]) {
  const int lane = threadIdx.x & 31;
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 16; ++k) stage[k * kStageStride + lane] = w[k];
  __syncwarp();
  const uint32_t* col = stage + (lane >> 1) * kStageStride;
  const uint32_t sel = (lane & 1) ? 0x7632u : 0x5410u;  // high or low halves of two words
  uint32_t o[16];
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint4 v = *reinterpret_cast<const uint4*>(col + 4 * q);
    o[2 * q] = __byte_perm(v.x, v.y, sel);
    o[2 * q + 1] = __byte_perm(v.z, v.w, sel);
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out_t) + static_cast<int64_t>(n + lane) * p.ld_t +
                                        (m - lane));
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
}

// The second operand an epilogue reads for row m, columns n .. n+31: U
// (kEpiGeluBwd, fp16) or the residual (kEpiResidual, bf16 or fp32) - 64 or
// 128 bytes, at the row stride ldo.  The epilogue loops load it one chunk
// ahead, while the current chunk is processed.
__device__ __forceinline__ bool epilogue_has_aux(const GemmParams& p) {
  return p.epi == kEpiGeluBwd || p.epi == kEpiResidual;
}

__device__ __forceinline__ void load_epilogue_aux(const GemmParams& p, int m, int n, uint4 (&a)[8]) {
  const int64_t off = static_cast<int64_t>(m) * p.ldo + n;
  if (p.epi == kEpiResidual && p.resid_f32) {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const float*>(p.resid) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = src[i];
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(p.resid) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = src[i];
  }
}

// kEpiResidual: accumulator values r plus the residual held in aux (fp32 or
// bf16), for one row's 32-column chunk.
__device__ __forceinline__ void residual_add(const GemmParams& p, const uint32_t (&r)[32], const uint4 (&aux)[8],
                                             float (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  if (p.resid_f32) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint4 q = aux[i];
      v[4 * i] += __uint_as_float(q.x); v[4 * i + 1] += __uint_as_float(q.y);
      v[4 * i + 2] += __uint_as_float(q.z); v[4 * i + 3] += __uint_as_float(q.w);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = aux[i];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 b2 = *reinterpret_cast<const __nv_bfloat162*>(&w[j]);
        const float2 f = __bfloat1622float2(b2);
        v[8 * i + 2 * j] += f.x;
        v[8 * i + 2 * j + 1] += f.y;
      }
    }
  }
}

// One 32 x 32 block of a residual epilogue - a warp's rows m0 .. m0+31 (lane
// = row), columns n .. n+31 - written by a tensor store.  Each lane puts its
// row into `buf` (4 KiB, 1024-byte aligned) in the layout of p.map_out's
// swizzle: 16-byte piece j of row i at piece j ^ (i & 7) of a 128-byte row
// (fp32) or j ^ ((i >> 1) & 3) of a 64-byte row (bf16), so eight consecutive
// lanes cover all 32 banks.  Lane 0 then stores the box.  The caller
// alternates two buffers per warp: before refilling one, lane 0 waits until
// at most its latest store (the other buffer's) is still reading.  The block
// lies wholly inside the output.
__device__ __forceinline__ void residual_chunk_tma(const GemmParams& p, int m0, int n, const uint32_t (&r)[32],
                                                   const uint4 (&aux)[8], uint8_t* buf) {
  const int lane = threadIdx.x & 31;
  if (!dbg_ok(m0 >= 0 && m0 + 32 <= p.M && n + 32 <= p.N, p.status)) return;
  float v[32];
  residual_add(p, r, aux, v);
  if (lane == 0) bulk_wait_group_read1();
  __syncwarp();
  if (p.out_f32) {
    uint8_t* row = buf + lane * 128;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      *reinterpret_cast<float4*>(row + ((j ^ (lane & 7)) << 4)) =
          make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
  } else {
    uint8_t* row = buf + lane * 64;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      *reinterpret_cast<uint4*>(row + ((j ^ ((lane >> 1) & 3)) << 4)) =
          make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                     pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
  }
  fence_proxy_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_2d(&p.map_out, buf, n, m0);
    bulk_commit_group();
  }
}

// One 32-column chunk of an output tile's epilogue: accumulator values r for
// local row m (global zigzag row grow) and output columns n .. n+31.
__device__ __forceinline__ void gemm_epilogue_chunk(const GemmParams& p, int m, int64_t grow, int n,
                                                    const uint32_t (&r)[32], const uint4 (&aux)[8],
                                                    uint32_t* stage) {
  if (!dbg_ok(m < p.M && n + 32 <= p.N, p.status)) return;
  if (p.epi == kEpiStoreF32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out[0]) + static_cast<int64_t>(m) * p.ldo + n);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]), __uint_as_float(r[4 * i + 2]),
                           __uint_as_float(r[4 * i + 3]));
    return;
  }
  if (p.epi == kEpiGeluBwd) {
    const int64_t off = static_cast<int64_t>(m) * p.ldo + n;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out[0]) + off);
    uint32_t tw[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 q = aux[i];
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 uf = __half22float2(*reinterpret_cast<const __half2*>(&w[j]));
        o[j] = pack_bf16x2(__uint_as_float(r[8 * i + 2 * j]) * gelu_tanh_grad_f(uf.x),
                           __uint_as_float(r[8 * i + 2 * j + 1]) * gelu_tanh_grad_f(uf.y));
      }
      dst[i] = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
      for (int j = 0; j < 4; ++j) tw[4 * i + j] = o[j];
    }
    if (p.out_t) store_transposed_bf16(p, stage, m, n, tw);
    return;
  }
  if (p.epi == kEpiResidual) {
    float v[32];
    residual_add(p, r, aux, v);
    const int64_t off = static_cast<int64_t>(m) * p.ldo + n;
    if (p.out_f32) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.out[0]) + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out[0]) + off);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        dst[i] = make_uint4(pack_bf16x2(v[8 * i], v[8 * i + 1]), pack_bf16x2(v[8 * i + 2], v[8 * i + 3]),
                            pack_bf16x2(v[8 * i + 4], v[8 * i + 5]), pack_bf16x2(v[8 * i + 6], v[8 * i + 7]));
    }
  } else {
    const int seg = n / p.seg_n;
    const int col = n - seg * p.seg_n;
    const int64_t orow = p.remap[seg] ? grow : m;
    if (!dbg_ok(seg < 3 && col + 32 <= p.seg_n && (!p.remap[seg] || (orow >= 0 && orow < p.remap_rows)), p.status))
      return;
    uint32_t packed[16];
    float mx = 0.f;  // largest magnitude converted: flags a saturation
    if (p.epi == kEpiGeluF16) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = gelu_tanh_f(__uint_as_float(r[2 * i])), b = gelu_tanh_f(__uint_as_float(r[2 * i + 1]));
        mx = fmax3(mx, fabsf(a), fabsf(b));
        packed[i] = pack_half2(a, b);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float a = __uint_as_float(r[2 * i]), b = __uint_as_float(r[2 * i + 1]);
        mx = fmax3(mx, fabsf(a), fabsf(b));
        packed[i] = pack_half2(a, b);
      }
    }
    note_fp16_saturation(p.status, mx);
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__half*>(p.out[seg]) + orow * p.ldo + col);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    if (p.out_t) {  // bf16(GELU(fp16 value)), transposed
      uint32_t tw[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&packed[i]));
        tw[i] = pack_bf16x2(gelu_tanh_f(f.x), gelu_tanh_f(f.y));
      }
      store_transposed_bf16(p, stage, m, n, tw);
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_f16_tcgen05(const __grid_constant__ GemmParams p) {
  using S = GemmShape<BN>;
  constexpr int STAGES = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * S::kBBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* tfull = bars + 2 * STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  const int num_m = (p.M + kGemmBM - 1) / kGemmBM;
  const int num_n = p.N / BN;
  const int num_k = p.K / kGemmBK;
  const int num_tiles = num_m * num_n;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&p.map_a);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, par = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        int mb, nb;
        gemm_tile_coords(tile, num_m, num_n, mb, nb);
        const int n0 = nb * BN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], S::kABytes + S::kBBytes);
          tma_load_2d(sA + stage * S::kABytes, &p.map_a, &full[stage], kb * kGemmBK, mb * kGemmBM);
          const CUtensorMap* mb_map;
          int bx, by;
          if (p.ksplit) {
            const int k0 = kb * kGemmBK;
            mb_map = &p.map_b[k0 / p.shard_k];
            bx = k0 % p.shard_k;
            by = n0;
          } else {
            mb_map = &p.map_b[n0 / p.shard_n];
            bx = kb * kGemmBK;
            by = n0 % p.shard_n;
          }
          tma_load_2d(sB + stage * S::kBBytes, mb_map, &full[stage], bx, by);
          used |= 1u << stage;
          par = (par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // every copy this thread started lands before the CTA exits
      for (int s = 0; s < STAGES; ++s)
        if (used & (1u << s)) mbar_drain(&full[s], (par >> s) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = p.fmt_bf16 ? idesc_f32acc(kGemmBM, BN, 0, 0, kFmtBF16)
                                        : idesc_f32acc(kGemmBM, BN, 0, 0, kFmtF16);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++acc) {
        const int buf = acc & 1;
        const uint32_t aph = (acc >> 1) & 1;
        if (!mbar_wait(&tempty[buf], aph ^ 1, ctl)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * BN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk) {
            const uint64_t ad = smem_desc_sw128(a0 + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(b0 + kk * 32, 16, 1024);
            mma_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0);
          }
          mma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) mma_commit(&tfull[buf]);
      }
      mma_commit(drain);
      mbar_drain(drain, 0, p.timeout_ns);
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters 2,3,0,1
    const int quarter = warp & 3;
    uint32_t* stage = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(bars) + S::kBarBytes) +
                      (warp - 2) * kStageWords;  // this warp's transpose buffer
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++acc) {
      int mb, nb;
      gemm_tile_coords(tile, num_m, num_n, mb, nb);
      const int buf = acc & 1;
      const uint32_t aph = (acc >> 1) & 1;
      if (!mbar_wait(&tfull[buf], aph, ctl)) break;
      tc_fence_after();
      const int m = mb * kGemmBM + row;
      const bool valid = m < p.M;
      const int64_t grow = (m < p.c) ? (p.off0 + m) : (p.off1 + m);
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t r[32];
        __syncwarp();
        tmem_ld32(tmem_base + lane_off + buf * BN + ch * 32, r);
        tmem_ld_wait();
        reg_fence32(r);
        const int n = nb * BN + ch * 32;
        uint4 aux[8] = {};
        if (valid && epilogue_has_aux(p)) load_epilogue_aux(p, m, n, aux);
        if (valid) gemm_epilogue_chunk(p, m, grow, n, r, aux, stage);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, S::kTmemCols);
  }
}

}  // namespace tsp
