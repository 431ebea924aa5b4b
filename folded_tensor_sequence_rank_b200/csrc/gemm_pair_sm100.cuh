// gemm_pair_sm100.cuh - the TSP shard-loop GEMM of gemm_sm100.cuh with
// 256 x 256 output tiles computed by a pair of CTAs on two SMs
// (tcgen05.mma.cta_group::2, M = 256).
//
// Why pairs: a 128 x 256 tile per SM streams (128 + 256) x 64 fp16 = 48 KiB of
// operands per 64-deep k-block, 96 B per clock at the tensor core's full
// rate, more than the ~50-65 B per clock per SM the L2 -> SM path delivers
// when every SM streams.  In a pair each SM loads its own 128 rows of A and
// half (128 rows) of the 256-row B tile: 32 KiB per k-block, 64 B per clock,
// and each operand byte feeds twice the MMA work.
//
// Same contract as gemm_f16_tcgen05 (GemmParams, N-split or K-split
// shard loop, epilogues): the even CTA of each pair (cluster rank 0) issues
// the MMAs; both CTAs run a TMA producer for their halves and an epilogue for
// their 128 rows.  Tile loads complete on the even CTA's barriers (TMA
// .cta_group::2), which the even producer arms with both CTAs' bytes; the MMA
// issuer's commits arrive on both CTAs' barriers (multicast); the odd CTA's
// epilogue warps free an accumulator by arriving remotely on the even CTA's
// barrier.  B maps have 128-row boxes (each CTA's half of a tile).
//
// Roles (192 threads per CTA, one CTA per SM, persistent over tile pairs):
//   warp 0     TMA producer (this CTA's A rows and B half)
//   warp 1     TMEM allocator (pair allocation); even CTA: MMA issuer
//   warps 2-5  epilogue of this CTA's 128 rows (TMEM lane quarters 2,3,0,1)
//
// Residual epilogues (the K-split GEMMs' output plus the residual stream)
// stage each warp's 32 x 32 output blocks in shared memory and write them with
// tensor stores, whole 128- or 64-byte rows at a time, instead of a lane per
// row storing 16 bytes to 32 different rows per instruction (which made the
// O projection at 16384 x 4096 x 4096 about 7% slower).  A warp whose rows
// run past M keeps the per-lane stores.
#pragma once
#include "gemm_sm100.cuh"
#include "ptx.cuh"

namespace tsp {

constexpr int kPairBM = 256;  // output rows per pair tile (128 per CTA)
constexpr int kPairBN = 256;

struct GemmPairShape {
  static constexpr int kABytes = 128 * kGemmBK * 2;  // this CTA's A rows: 16 KiB
  static constexpr int kBBytes = 128 * kGemmBK * 2;  // this CTA's half of B: 16 KiB
  static constexpr int kStages = 6;
  static constexpr int kTmemCols = 2 * kPairBN;  // two accumulators of 256 columns
  static constexpr int kBarBytes = 256;
  // per epilogue warp 8 KiB: two 4 KiB staging buffers of the tensor-store
  // epilogue, or the transpose buffer of the transposed bf16 stores
  static constexpr int kEpiWarpBytes = 8192;
  static constexpr int kEpiBytes = 4 * kEpiWarpBytes;
  static constexpr int kSmemBytes = kStages * (kABytes + kBBytes) + kEpiBytes + kBarBytes + 1024;
  static_assert(kStageWords * 4 <= kEpiWarpBytes, "transpose buffer fits the warp's staging");
  static_assert(kSmemBytes <= 232448, "shared memory of one CTA");
};

__global__ void __launch_bounds__(kGemmThreads, 1) gemm_pair_f16_tcgen05(const __grid_constant__ GemmParams p) {
  using S = GemmPairShape;
  constexpr int STAGES = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * S::kABytes;
  uint8_t* sEpi = sB + STAGES * S::kBBytes;  // 1024-byte aligned
  uint64_t* bars = reinterpret_cast<uint64_t*>(sEpi + S::kEpiBytes);
  uint64_t* full = bars;               // [STAGES] even CTA: both CTAs' tiles landed
  uint64_t* empty = full + STAGES;     // [STAGES] both CTAs: MMAs done with the stage
  uint64_t* tfull = empty + STAGES;    // [2] both CTAs: accumulator holds a finished tile
  uint64_t* tempty = tfull + 2;        // [2] even CTA: both epilogues have read it (4 warps x 2 CTAs)
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t cta = cluster_ctarank();

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 8);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc2(tmem_slot, S::kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers initialised and tensor memory allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  const int num_m = (p.M + kPairBM - 1) / kPairBM;
  const int num_n = p.N / kPairBN;
  const int num_k = p.K / kGemmBK;
  const int num_tiles = num_m * num_n;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (elect_one()) {
      tma_prefetch_desc(&p.map_a);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t used = 0, par = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += npairs) {
        int mb, nb;
        gemm_tile_coords(tile, num_m, num_n, mb, nb);
        const int n0 = nb * kPairBN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, ctl)) { ok = false; break; }
          if (cta == 0) mbar_arrive_expect_tx(&full[stage], 2 * (S::kABytes + S::kBBytes));
          const uint32_t fb = mapa_shared(smem_u32(&full[stage]), 0);
          tma2_load_2d(sA + stage * S::kABytes, &p.map_a, fb, kb * kGemmBK,
                       mb * kPairBM + 128 * static_cast<int>(cta));
          const CUtensorMap* b_map;
          int bx, by;
          if (p.ksplit) {
            const int k0 = kb * kGemmBK;
            b_map = &p.map_b[k0 / p.shard_k];
            bx = k0 % p.shard_k;
            by = n0;
          } else {
            b_map = &p.map_b[n0 / p.shard_n];
            bx = kb * kGemmBK;
            by = n0 % p.shard_n;
          }
          tma2_load_2d(sB + stage * S::kBBytes, b_map, fb, bx, by + 128 * static_cast<int>(cta));
          used |= 1u << stage;
          par = (par & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the even CTA's full barriers count both CTAs' bytes: draining them
      // waits for every copy of the pair
      if (cta == 0)
        for (int s = 0; s < STAGES; ++s)
          if (used & (1u << s)) mbar_drain(&full[s], (par >> s) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    if (cta == 0 && elect_one()) {
      const uint32_t idesc = p.fmt_bf16 ? idesc_f32acc(kPairBM, kPairBN, 0, 0, kFmtBF16)
                                        : idesc_f32acc(kPairBM, kPairBN, 0, 0, kFmtF16);
      constexpr uint16_t kBoth = 3;
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      bool ok = true;
      for (int tile = pair; ok && tile < num_tiles; tile += npairs, ++acc) {
        const int buf = acc & 1;
        const uint32_t aph = (acc >> 1) & 1;
        if (!mbar_wait_cl(&tempty[buf], aph ^ 1, ctl)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kPairBN;
        for (int kb = 0; kb < num_k; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * S::kABytes);
          const uint32_t b0 = smem_u32(sB + stage * S::kBBytes);
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            mma2_ss(d_tmem, smem_desc_sw128(a0 + kk * 32, 16, 1024), smem_desc_sw128(b0 + kk * 32, 16, 1024), idesc,
                    (kb | kk) != 0);
          mma2_commit_mc(&empty[stage], kBoth);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) mma2_commit_mc(&tfull[buf], kBoth);
      }
      mma2_commit_mc(drain, 1);
      mbar_drain(drain, 0, p.timeout_ns);
    }
  } else {
    // epilogue warps 2..5 -> TMEM lane quarters 2,3,0,1 of this CTA's 128 rows
    const int quarter = warp & 3;
    uint8_t* wstage = sEpi + (warp - 2) * S::kEpiWarpBytes;  // this warp's staging
    uint32_t* stage = reinterpret_cast<uint32_t*>(wstage);     // as the transpose buffer
    const int row = quarter * 32 + lane;
    int staged = 0;  // tensor-store blocks this warp has issued: picks the buffer
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    int acc = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs, ++acc) {
      int mb, nb;
      gemm_tile_coords(tile, num_m, num_n, mb, nb);
      const int buf = acc & 1;
      const uint32_t aph = (acc >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], aph, ctl))) break;
      tc_fence_after();
      const int m = mb * kPairBM + 128 * static_cast<int>(cta) + row;
      const bool valid = m < p.M;
      // the warp's 32 rows go out by tensor stores when they all exist
      const int m0w = m - lane;
      const bool tma_rows = p.tma_out && m0w + 32 <= p.M;
      const int64_t grow = (m < p.c) ? (p.off0 + m) : (p.off1 + m);
      // Software-pipelined over the 32-column chunks: the next chunk's
      // accumulators (and its U values or residual) are loaded while this
      // chunk is processed.
      constexpr int kChunks = kPairBN / 32;
      const bool aux_on = valid && epilogue_has_aux(p);
      uint32_t r[32], rn[32];
      uint4 aux[8] = {}, auxn[8] = {};
      __syncwarp();
      tmem_ld32(tmem_base + lane_off + buf * kPairBN, r);
      if (aux_on) load_epilogue_aux(p, m, nb * kPairBN, aux);
      tmem_ld_wait();
      reg_fence32(r);
#pragma unroll 1
      for (int ch = 0; ch < kChunks; ++ch) {
        if (ch + 1 < kChunks) {
          __syncwarp();
          tmem_ld32(tmem_base + lane_off + buf * kPairBN + (ch + 1) * 32, rn);
          if (aux_on) load_epilogue_aux(p, m, nb * kPairBN + (ch + 1) * 32, auxn);
        }
        if (tma_rows)
          residual_chunk_tma(p, m0w, nb * kPairBN + ch * 32, r, aux, wstage + (staged++ & 1) * 4096);
        else if (valid)
          gemm_epilogue_chunk(p, m, grow, nb * kPairBN + ch * 32, r, aux, stage);
        if (ch + 1 < kChunks) {
          tmem_ld_wait();
          reg_fence32(rn);  // no use of rn before the wait
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = rn[i];
#pragma unroll
          for (int i = 0; i < 8; ++i) aux[i] = auxn[i];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&tempty[buf]), 0));
    }
    // the tensor stores have read the staging and written the output before
    // the CTA's shared memory is released
    if (lane == 0 && staged) bulk_wait_group0();
  }

  // the MMA issuer may still write the odd CTA's tensor memory, and the odd
  // CTA arrive on the even CTA's barriers, until both CTAs are here
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc2(tmem_base, S::kTmemCols);
  }
}

}  // namespace tsp
