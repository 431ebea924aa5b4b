// attn_bwd_sm100.cuh - backward of one TSP rank's causal attention against the
// all-gathered full-sequence K/V, for sm_100a tensor cores.
//
// What it computes (the chain rule through the forward of attn_sm100.cuh; the
// TSP news item, zubnet.ai, paragraph 1 gives training as the workload and
// paragraph 2 the all-gathered K/V, so a rank's dK/dV for ALL keys go back to
// the key owners, summed over ranks): per head, for the rank's query rows i
// at global positions p(i) and keys k <= p(i),
//     P   = 2^(s * scale * log2 e - lse2)      (lse2 stashed by the forward)
//     dP  = dO V^T,   Delta_i = sum_c dO_ic O_ic
//     dS  = scale * P * (dP - Delta)
//     dV += P^T dO,   dK += dS^T Q,   dQ += dS K.
// Key tiles are the outer loop: a work item is (head, 128-key tile), which
// loops over every 128-row query tile of the rank that reaches that key tile
// (query tiles lie inside one zigzag chunk; a tile reaches key tile kt if its
// last position is >= kt * 128).  dK and dV of the key tile accumulate in
// tensor memory over the item and are added to the caller's full-sequence
// dK, dV at the end of the item; each query tile's dQ contribution is added
// to the rank's dQ (fp32) with vector reductions, since every key tile adds to
// the same rows.  Items go out through an atomic counter, head-major with the
// heaviest key tiles of a head first (key tile kt is reached by every query
// tile that reaches kt + 1).
//
// Roles (384 threads = three warpgroups, one CTA per SM, persistent):
//   warp 0      work queue + TMA producer: K, V of the item; Q, lse2, Delta
//               (2-stage ring) and dO (1 stage) of each query tile
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-3   idle (they complete the first warpgroup)
//   warps 4-11  elementwise softmax gradient, dQ read-out, dK/dV epilogue; a
//               thread owns one key row (TMEM lane) and half of the columns,
//               so two warps share each lane quarter
// As in the forward kernel the registers are re-split at the start
// (setmaxnreg): kBwdLowRegs for the first warpgroup, kBwdHighRegs for the
// two softmax warpgroups, within the 168 per thread of the launch.
// Tensor memory (512 columns): [dK | dV | S^T | dP^T] = 128 each (dK, dV use
// head_dim of their 128).  Per query tile:
//   S^T = K Q^T  and  dP^T = V dO^T  (keys on the lanes; SS MMAs, K-major);
//   the softmax warps read S^T and dP^T, write P^T as fp16 pairs into the
//   dP^T columns they have read (TS operand of dV) and dS^T as fp16 into
//   shared memory in the 128-byte swizzled layout that is at once a K-major
//   operand [keys x queries] (for dK) and an MN-major operand [queries x
//   keys] (for dQ);
//   dV += P^T dO (TS, dO MN-major), dK += dS^T Q (SS, Q MN-major), and, once
//   the dV MMA has completed (it reads P^T from the dP^T columns), dQ = dS K
//   into the dP^T columns (SS, both MN-major); the softmax warps read dQ out
//   of tensor memory (which frees the columns at once) and add it to global
//   memory: each warp stages its 32 x 32 fp32 blocks in its 4 KiB of the dS^T
//   buffer (and a second 4 KiB block at head_dim 128) and one lane adds each
//   block with a TMA bulk reduction (whole 128-byte lines per L2 operation
//   instead of 16-byte vector reductions); the next tile's dS^T stores wait
//   until those reductions have read the staging.
// Q, K, V, dO, P and dS are fp16 (the forward's operand format); scores,
// statistics, accumulators and the outputs are fp32.
#pragma once
#include "attn_sm100.cuh"
#include "misc_kernels.cuh"
#include "ptx.cuh"

namespace tsp {

constexpr int kBwdThreads = 384;        // three warpgroups
constexpr int kBwdLaunchRegs = 168;     // per thread at launch: 65536 / 384, rounded down to 8
constexpr int kBwdLowRegs = 80;         // warps 0-3 after the re-split
constexpr int kBwdHighRegs = 208;       // the softmax warpgroups after the re-split
static_assert(128 * kBwdLowRegs + 256 * kBwdHighRegs <= kBwdThreads * kBwdLaunchRegs, "register split");
constexpr int kBwdTile = 128;  // keys per item, queries per query tile

struct __align__(64) AttnBwdParams {
  CUtensorMap map_q;   // Q [L, h] fp16, box {64, 128}
  CUtensorMap map_do;  // dO [L, h] fp16, box {64, 128}
  CUtensorMap map_k;   // K [T, h] fp16, box {64, 128}
  CUtensorMap map_v;   // V [T, h] fp16, box {64, 128}
  CUtensorMap map_dq;  // dQ [L, h] fp32, box {32, 32}, 128-byte swizzle (bulk reductions)
  const float* lse;    // [H][2][c_pad] log2-domain log-sum-exp (forward stash)
  const float* delta;  // [H][2][c_pad] scale * rowsum(dO * O) per head
  float* dq;           // [L, h] fp32, added to
  float* dk;           // [T, h] fp32, added to
  float* dv;           // [T, h] fp32, added to
  int64_t ld;          // h
  int64_t T;
  int c, c_pad, rank, D, H;
  int nqt;             // query tiles per chunk
  int nkt;             // key tiles: ceil(last position of the rank + 1, 128)
  int n_items;         // H * nkt
  float scale_log2;    // softmax scale * log2(e)
  float scale;         // softmax scale
  int* counter;        // work queue head (zeroed before launch)
  int* status;
  uint64_t timeout_ns;
};

template <int HD>
struct AttnBwdShape {
  static constexpr int kTileBytes = kBwdTile * HD * 2;  // one 128-row fp16 tile
  static constexpr int kStatBytes = kBwdTile * 4;       // lse2 or Delta of one query tile
  static constexpr int kQStages = 2;
  static constexpr int kBarBytes = 512;
  // second staging block per softmax warp (head_dim 128: its 64 columns of a
  // dQ row are two 32-column blocks; the first is staged in the dS^T buffer)
  static constexpr int kStage2Bytes = HD == 128 ? 8 * 4096 : 0;
  // K, V, dO, dS^T (128 x 128 whatever the head size), the Q ring, the second
  // staging blocks, the Q ring's statistics.  The dynamic shared memory base
  // is 1024-byte aligned (checked at run time), so no slack is added.
  static constexpr int kSmemBytes =
      3 * kTileBytes + 32768 + kQStages * kTileBytes + kStage2Bytes + kQStages * 2 * kStatBytes + kBarBytes;
};

struct BwdQTile {
  int m0;      // first local row
  int p0;      // global position of the first row
  int nvalid;  // rows inside the chunk
  int chunk;   // 0: chunk r, 1: chunk 2D-1-r
  int t;       // tile index inside the chunk
};

// Query tile n (0 .. 2*nqt-1) of the rank: chunk 2D-1-r first (the tiles that
// reach the most key tiles), then chunk r.
__device__ __forceinline__ BwdQTile bwd_qtile(const AttnBwdParams& p, int n) {
  BwdQTile q;
  q.chunk = n < p.nqt ? 1 : 0;
  q.t = n < p.nqt ? n : n - p.nqt;
  const int gchunk = q.chunk ? (2 * p.D - 1 - p.rank) : p.rank;
  q.m0 = q.chunk * p.c + q.t * kBwdTile;
  q.p0 = gchunk * p.c + q.t * kBwdTile;
  q.nvalid = min(kBwdTile, p.c - q.t * kBwdTile);
  return q;
}

__device__ __forceinline__ bool bwd_reaches(const BwdQTile& q, int kt) {
  return q.p0 + q.nvalid - 1 >= kt * kBwdTile;
}

// Offset (bytes) of the 16-byte group holding columns 8j .. 8j+7 of row r in
// a 128-row tile stored as 64-column boxes of 128-byte rows with the 128-byte
// swizzle (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B).
__device__ __forceinline__ uint32_t sw128_offset(int r, int j) {
  return static_cast<uint32_t>((j >> 3) * 16384 + r * 128 + (((j & 7) ^ (r & 7)) << 4));
}

template <int HD>
__global__ void __launch_bounds__(kBwdThreads, 1) attn_bwd_tcgen05(const __grid_constant__ AttnBwdParams p) {
  using S = AttnBwdShape<HD>;
  constexpr int NB = HD / 64;  // 64-column boxes per tile row
  constexpr int QST = S::kQStages;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // The 128-byte swizzle needs 1024-byte aligned tiles; the dynamic shared
  // memory base is (0x400 on this GPU), and the size has no slack for a
  // misaligned one: such a launch records the failed check and does nothing.
  if (smem_u32(smem_raw) & 1023) {
    if (threadIdx.x == 0) atomicOr(p.status + 1, kFlagBoundsCheck);
    return;
  }
  uint8_t* smem = smem_raw;
  uint8_t* sK = smem;
  uint8_t* sV = sK + S::kTileBytes;
  uint8_t* sDO = sV + S::kTileBytes;
  uint8_t* sDS = sDO + S::kTileBytes;  // dS^T [128 keys][128 queries] fp16: always 2 boxes of 64 queries
  uint8_t* sQ = sDS + 32768;           // [QST][kTileBytes]
  uint8_t* sStage2 = sQ + QST * S::kTileBytes;  // [8 warps][4 KiB] (head_dim 128)
  float* sStat = reinterpret_cast<float*>(sStage2 + S::kStage2Bytes);  // [QST][lse2 | Delta][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStat + QST * 2 * kBwdTile);
  uint64_t* kv_full = bars;           // K, V of the item landed
  uint64_t* kv_empty = kv_full + 1;   // the item's last MMA reading K, V done
  uint64_t* q_full = kv_empty + 1;    // [QST] Q tile + statistics landed
  uint64_t* q_empty = q_full + QST;   // [QST]
  uint64_t* do_full = q_empty + QST;
  uint64_t* do_empty = do_full + 1;
  uint64_t* s_full = do_empty + 1;    // S^T, dP^T in tensor memory
  uint64_t* p_full = s_full + 1;      // P^T (tensor memory) and dS^T (shared) written, 8 warps
  uint64_t* dv_done = p_full + 1;     // the dV MMA of the tile completed
  uint64_t* dq_full = dv_done + 1;    // dQ of the tile in tensor memory
  uint64_t* dq_free = dq_full + 1;    // dQ read out of tensor memory, 8 warps
  uint64_t* stg_free = dq_free + 1;   // every warp's staged dQ blocks have been read, 8 warps
  uint64_t* dkv_full = stg_free + 1;  // dK, dV of the item complete
  uint64_t* dkv_free = dkv_full + 1;  // dK, dV read out, 8 warps
  uint64_t* it_full = dkv_free + 1;   // [2]
  uint64_t* it_empty = it_full + 2;   // [2]
  uint64_t* drain = it_empty + 2;
  int* it_slot = reinterpret_cast<int*>(drain + 1);  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(it_slot + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 8);
    mbar_init(dv_done, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 8);
    mbar_init(stg_free, 8);
    mbar_init(dkv_full, 1);
    mbar_init(dkv_free, 8);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&it_full[x], 1);
      mbar_init(&it_empty[x], 9);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t t_dk = tmem, t_dv = tmem + 128, t_s = tmem + 256, t_dp = tmem + 384;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};
  const int nq_all = 2 * p.nqt;

  if (warp < 4) {
    __syncwarp();
    regs_dec<kBwdLowRegs>();
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      tma_prefetch_desc(&p.map_q);
      tma_prefetch_desc(&p.map_do);
      tma_prefetch_desc(&p.map_k);
      tma_prefetch_desc(&p.map_v);
      uint32_t kvph = 0, doph = 0, qph[QST] = {0, 0};
      int qs = 0;
      bool kv_used = false, do_used = false;
      uint32_t kv_par = 0, do_par = 0, q_used = 0, q_par = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait_inl(&it_empty[slot], ((n >> 1) & 1) ^ 1, ctl)) break;
        int it = atomicAdd(p.counter, 1);
        if (it >= p.n_items) it = -1;
        it_slot[slot] = it;
        mbar_arrive(&it_full[slot]);
        if (it < 0) break;
        const int head = it / p.nkt, kt = it % p.nkt;
        const int col0 = head * HD;
        if (!mbar_wait_inl(kv_empty, kvph ^ 1, ctl)) break;
        mbar_arrive_expect_tx(kv_full, 2 * S::kTileBytes);
#pragma unroll
        for (int b = 0; b < NB; ++b) {
          tma_load_2d(sK + b * 16384, &p.map_k, kv_full, col0 + 64 * b, kt * kBwdTile);
          tma_load_2d(sV + b * 16384, &p.map_v, kv_full, col0 + 64 * b, kt * kBwdTile);
        }
        kv_used = true;
        kv_par = kvph;
        kvph ^= 1;
        for (int n2 = 0; ok && n2 < nq_all; ++n2) {
          const BwdQTile q = bwd_qtile(p, n2);
          if (!bwd_reaches(q, kt)) continue;
          if (!mbar_wait_inl(&q_empty[qs], qph[qs] ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[qs], S::kTileBytes + 2 * S::kStatBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sQ + qs * S::kTileBytes + b * 16384, &p.map_q, &q_full[qs], col0 + 64 * b, q.m0);
          const int64_t srow = static_cast<int64_t>(head * 2 + q.chunk) * p.c_pad + q.t * kBwdTile;
          if (!dbg_ok(q.t * kBwdTile + kBwdTile <= p.c_pad && head < p.H, p.status)) { ok = false; break; }
          bulk_load(sStat + qs * 2 * kBwdTile, p.lse + srow, S::kStatBytes, &q_full[qs]);
          bulk_load(sStat + qs * 2 * kBwdTile + kBwdTile, p.delta + srow, S::kStatBytes, &q_full[qs]);
          q_used |= 1u << qs;
          q_par = (q_par & ~(1u << qs)) | (qph[qs] << qs);
          qph[qs] ^= 1;
          if (++qs == QST) qs = 0;
          if (!mbar_wait_inl(do_empty, doph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(do_full, S::kTileBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b) tma_load_2d(sDO + b * 16384, &p.map_do, do_full, col0 + 64 * b, q.m0);
          do_used = true;
          do_par = doph;
          doph ^= 1;
        }
      }
      // every copy this thread started lands before the CTA exits
      if (kv_used) mbar_drain(kv_full, kv_par, p.timeout_ns);
      if (do_used) mbar_drain(do_full, do_par, p.timeout_ns);
      for (int s = 0; s < QST; ++s)
        if (q_used & (1u << s)) mbar_drain(&q_full[s], (q_par >> s) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_f32acc(kBwdTile, kBwdTile, 0, 0, kFmtF16);  // S^T, dP^T
      constexpr uint32_t idesc_kv = idesc_f32acc(kBwdTile, HD, 0, 1, kFmtF16);       // dV (TS), dK
      constexpr uint32_t idesc_q = idesc_f32acc(kBwdTile, HD, 1, 1, kFmtF16);        // dQ
      // K-major descriptors of K, V, dO, Q (scores) and dS^T (dK); MN-major of
      // dO, Q (dV, dK), dS (dQ) and K (dQ).
      const uint64_t dK_k = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t dV_k = smem_desc_sw128(smem_u32(sV), 16, 1024);
      const uint64_t dDO_k = smem_desc_sw128(smem_u32(sDO), 16, 1024);
      const uint64_t dQ_k0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t dDS_k = smem_desc_sw128(smem_u32(sDS), 16, 1024);
      const uint64_t dDO_mn = smem_desc_sw128(smem_u32(sDO), 16384, 1024);
      const uint64_t dQ_mn0 = smem_desc_sw128(smem_u32(sQ), 16384, 1024);
      const uint64_t dDS_mn = smem_desc_sw128(smem_u32(sDS), 16384, 1024);
      const uint64_t dK_mn = smem_desc_sw128(smem_u32(sK), 16384, 1024);
      uint32_t kvph = 0, doph = 0, qph[QST] = {0, 0};
      int qs = 0;
      uint32_t tiles = 0;  // query tiles processed (all items)
      uint32_t items = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait_inl(&it_full[slot], (n >> 1) & 1, ctl)) break;
        const int it = it_slot[slot];
        mbar_arrive(&it_empty[slot]);
        if (it < 0) break;
        const int kt = it % p.nkt;
        if (!mbar_wait_inl(kv_full, kvph, ctl)) break;
        kvph ^= 1;
        tc_fence_after();
        bool first = true;
        for (int n2 = 0; ok && n2 < nq_all; ++n2) {
          const BwdQTile q = bwd_qtile(p, n2);
          if (!bwd_reaches(q, kt)) continue;
          const uint64_t dQ_k = dQ_k0 + static_cast<uint64_t>(qs * (S::kTileBytes >> 4));
          const uint64_t dQ_mn = dQ_mn0 + static_cast<uint64_t>(qs * (S::kTileBytes >> 4));
          if (!mbar_wait_inl(&q_full[qs], qph[qs], ctl)) { ok = false; break; }
          tc_fence_after();
          // S^T = K Q^T (K = head_dim); the softmax warps read the previous
          // tile's S^T before they signalled p_full
          if constexpr (HD == 128) {
            mma_ss_x8<0, 2, 4, 6, 1024, 1026, 1028, 1030>(t_s, dK_k, dQ_k, idesc_s, 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) mma_ss(t_s, dK_k + 2 * kk, dQ_k + 2 * kk, idesc_s, kk != 0);
          }
          if (!mbar_wait_inl(do_full, doph, ctl)) { ok = false; break; }
          // dP^T = V dO^T: the dP^T columns hold the previous tile's dQ until
          // it is read out
          if (tiles > 0 && !mbar_wait_inl(dq_free, (tiles - 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          if constexpr (HD == 128) {
            mma_ss_x8<0, 2, 4, 6, 1024, 1026, 1028, 1030>(t_dp, dV_k, dDO_k, idesc_s, 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < HD / 16; ++kk) mma_ss(t_dp, dV_k + 2 * kk, dDO_k + 2 * kk, idesc_s, kk != 0);
          }
          mma_commit(s_full);
          if (!mbar_wait_inl(p_full, tiles & 1, ctl)) { ok = false; break; }
          // the first tile of an item overwrites dK, dV: the previous item's
          // epilogue must have read them
          if (first && items > 0 && !mbar_wait_inl(dkv_free, (items - 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          // dV += P^T dO: A = P^T from the dP^T columns (fp16 pairs; queries
          // 0-63 in columns 0-31, queries 64-127 in columns 64-95), B = dO
          // MN-major, 16 queries (2 KiB of dO) per step
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(t_dv, t_dp + (kk < 4 ? 8 * kk : 64 + 8 * (kk - 4)), dDO_mn + 128 * kk, idesc_kv,
                   (!first || kk != 0) ? 1u : 0u);
          mma_commit(dv_done);
          mma_commit(do_empty);
          // dK += dS^T Q: A = dS^T K-major (16 queries = 32 bytes per step, the
          // next 64 queries 16 KiB on), B = Q MN-major
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(t_dk, dDS_k + ((kk >> 2) * 1024 + (kk & 3) * 2), dQ_mn + 128 * kk, idesc_kv,
                   (!first || kk != 0) ? 1u : 0u);
          // dQ = dS K into the dP^T columns, once the dV MMA has read P^T
          if (!mbar_wait_inl(dv_done, tiles & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          mma_ss_x8<0, 128, 256, 384, 512, 640, 768, 896>(t_dp, dDS_mn, dK_mn, idesc_q, 0);
          mma_commit(dq_full);
          mma_commit(&q_empty[qs]);
          qph[qs] ^= 1;
          if (++qs == QST) qs = 0;
          doph ^= 1;
          ++tiles;
          first = false;
        }
        if (!ok) break;
        mma_commit(kv_empty);
        mma_commit(dkv_full);
        ++items;
      }
      mma_commit(drain);
      mbar_drain(drain, 0, p.timeout_ns);
    }
  }
  } else {
    // ---------------------------------------------------------------- softmax gradient
    __syncwarp();
    regs_inc<kBwdHighRegs>();
    const int quarter = warp & 3;       // TMEM lane quarter: key rows 32*quarter ..
    const int half = (warp - 4) >> 2;   // query columns 64*half .. 64*half+63
    const int kr = quarter * 32 + lane; // key row of this thread
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    const float2 sl2v = make_float2(sl2, sl2);
    const float2 scv = make_float2(p.scale, p.scale);
    uint32_t qph[QST] = {0, 0};
    int qs = 0;
    uint32_t tiles = 0, items = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int slot = n & 1;
      if (!warp_wait(&it_full[slot], (n >> 1) & 1, ctl)) break;
      const int it = it_slot[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&it_empty[slot]);
      if (it < 0) break;
      const int head = it / p.nkt, kt = it % p.nkt;
      const int kpos = kt * kBwdTile + kr;
      for (int n2 = 0; ok && n2 < nq_all; ++n2) {
        const BwdQTile q = bwd_qtile(p, n2);
        if (!bwd_reaches(q, kt)) continue;
        if (!warp_wait(&q_full[qs], qph[qs], ctl) || !warp_wait(s_full, tiles & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const float* st_lse = sStat + qs * 2 * kBwdTile;
        const float* st_dl = st_lse + kBwdTile;
        // columns valid for this key row: query q < nvalid and position
        // p0 + q >= kpos
        const int qmin = kpos - q.p0;  // <= 0: no causal mask on this row
        const bool full = qmin <= 0 && q.nvalid == kBwdTile;
        uint32_t P[32];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int col0 = half * 64 + cc * 32;
          uint32_t sr[32], dr[32];
          tmem_ld32(t_s + lane_off + col0, sr);
          tmem_ld32(t_dp + lane_off + col0, dr);
          tmem_ld_wait();
          reg_fence32(sr);
          reg_fence32(dr);
          uint32_t dsp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int qc = col0 + 2 * i;
            const float2 l2 = *reinterpret_cast<const float2*>(st_lse + qc);
            const float2 dl = *reinterpret_cast<const float2*>(st_dl + qc);
            const float2 xv = ffma2(make_float2(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), sl2v,
                                    make_float2(-l2.x, -l2.y));
            float2 pr;
            if ((i & 3) == 3) {
              pr = exp2_poly2(xv);
            } else {
              pr.x = ex2_approx(xv.x);
              pr.y = ex2_approx(xv.y);
            }
            // dS = P (scale dP - scale Delta); Delta arrives already scaled
            const float2 tv = ffma2(make_float2(__uint_as_float(dr[2 * i]), __uint_as_float(dr[2 * i + 1])), scv,
                                    make_float2(-dl.x, -dl.y));
            float2 dsv = fmul2(pr, tv);
            if (!full) {
              const bool v0 = qc >= qmin && qc < q.nvalid, v1 = qc + 1 >= qmin && qc + 1 < q.nvalid;
              pr.x = v0 ? pr.x : 0.f;
              pr.y = v1 ? pr.y : 0.f;
              dsv.x = v0 ? dsv.x : 0.f;
              dsv.y = v1 ? dsv.y : 0.f;
            }
            P[cc * 16 + i] = pack_half2(pr.x, pr.y);
            dsp[i] = pack_half2(dsv.x, dsv.y);
          }
          // dS^T row kr, queries col0 .. col0+31: four 16-byte groups.  The
          // buffer held the previous tile's staged dQ blocks: each warp waits
          // for its own bulk reductions to have read them, then for every
          // warp's (deferred to here, so the wait overlaps this softmax)
          if (cc == 0 && tiles > 0) {
            if (lane == 0) bulk_wait_group_read0();
            __syncwarp();
            if (lane == 0) mbar_arrive(stg_free);
            if (!warp_wait(stg_free, (tiles - 1) & 1, ctl)) { ok = false; break; }
          }
          uint8_t* rowp = sDS;
#pragma unroll
          for (int g = 0; g < 4; ++g)
            *reinterpret_cast<uint4*>(rowp + sw128_offset(kr, col0 / 8 + g)) =
                make_uint4(dsp[4 * g], dsp[4 * g + 1], dsp[4 * g + 2], dsp[4 * g + 3]);
        }
        if (!ok) break;
        // P^T over the dP^T columns this warp has read (queries 64*half ..)
        tmem_st32p(t_dp + lane_off + half * 64, P);
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full);
        // this tile's dQ: query rows on the lanes, head_dim columns split by half
        if (!warp_wait(dq_full, tiles & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        {
          // the whole of this warp's dQ block into registers, then the tensor
          // memory columns go back to the issuer
          uint32_t r[HD / 2];
#pragma unroll
          for (int j = 0; j < HD / 64; ++j) tmem_ld32p(t_dp + lane_off + half * (HD / 2) + 32 * j, &r[32 * j]);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < HD / 64; ++j) reg_fence32(&r[32 * j]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(dq_free);
          if (q.nvalid == kBwdTile) {
            // whole tile: stage each 32 x 32 block (128-byte swizzled) in this
            // warp's 4 KiB of the dS^T buffer - free: the dQ MMA has read it -
            // and, at head_dim 128, in its second block; one bulk reduction
            // adds each.  The reads of the staging are waited for just before
            // the next tile's dS^T stores.
#pragma unroll
            for (int j = 0; j < HD / 64; ++j) {
              uint8_t* stg = j == 0 ? sDS + (warp - 4) * 4096 : sStage2 + (warp - 4) * 4096;
#pragma unroll
              for (int c = 0; c < 8; ++c)
                *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                    make_uint4(r[32 * j + 4 * c], r[32 * j + 4 * c + 1], r[32 * j + 4 * c + 2], r[32 * j + 4 * c + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0 && dbg_ok(q.m0 + quarter * 32 + 32 <= 2 * p.c && (head + 1) * HD <= p.ld, p.status)) {
#pragma unroll
              for (int j = 0; j < HD / 64; ++j)
                tma_reduce_add_2d(&p.map_dq, j == 0 ? sDS + (warp - 4) * 4096 : sStage2 + (warp - 4) * 4096,
                                  head * HD + half * (HD / 2) + 32 * j, q.m0 + quarter * 32);
              bulk_commit_group();
            }
            __syncwarp();
          } else {
            // a ragged tile (the last of a chunk whose length is not a multiple
            // of 128): rows past the chunk are skipped, one vector reduction
            // per 16 bytes
            const int qrow = kr;  // lane = query row of the dQ tile
            if (qrow < q.nvalid && dbg_ok(q.m0 + qrow < 2 * p.c, p.status)) {
              float* dst = p.dq + static_cast<int64_t>(q.m0 + qrow) * p.ld + head * HD + half * (HD / 2);
#pragma unroll
              for (int i = 0; i < HD / 8; ++i)
                atomicAdd(reinterpret_cast<float4*>(dst) + i,
                          make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                      __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
            }
          }
        }
        qph[qs] ^= 1;
        if (++qs == QST) qs = 0;
        ++tiles;
      }
      if (!ok) break;
      // the item's dK, dV: key rows on the lanes, head_dim columns split by half
      if (!warp_wait(dkv_full, items & 1, ctl)) break;
      tc_fence_after();
      {
        // every lane takes part in the tensor-memory loads; keys past the
        // sequence (a partial last key tile) add nothing
        const bool kvalid = kpos < p.T;
        const int64_t off = static_cast<int64_t>(kvalid ? kpos : 0) * p.ld + head * HD + half * (HD / 2);
#pragma unroll
        for (int which = 0; which < 2; ++which) {
          float* dst = (which == 0 ? p.dk : p.dv) + off;
          const uint32_t src = (which == 0 ? t_dk : t_dv) + lane_off + half * (HD / 2);
#pragma unroll
          for (int j = 0; j < HD / 64; ++j) {
            uint32_t r[32];
            tmem_ld32(src + 32 * j, r);
            tmem_ld_wait();
            reg_fence32(r);
            if (kvalid && dbg_ok((head + 1) * HD <= p.ld, p.status)) {
#pragma unroll
              for (int i = 0; i < 8; ++i)
                atomicAdd(reinterpret_cast<float4*>(dst + 32 * j) + i,
                          make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                      __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3])));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dkv_free);
      ++items;
    }
  }

  // the CTA outlives the reads of its last bulk reductions
  if (warp >= 4 && lane == 0) bulk_wait_group_read0();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Delta = scale * rowsum over each head's columns of dO * O, written per
// head and chunk as [H][2][c_pad] (the layout of the forward's lse stash):
// one 256-thread block per local row, each thread 8 columns.
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_delta_kernel(const __half* __restrict__ dout,
                                                             const __half* __restrict__ out, float* __restrict__ delta,
                                                             int h, int c, int c_pad, float scale) {
  const int64_t row = blockIdx.x;
  constexpr int kLanesPerHead = HD / 8;
  // the same number of passes for every thread (the shuffles need the whole
  // warp); columns past h contribute nothing
  for (int base = 0; base < h; base += 256 * 8) {
    const int col = base + threadIdx.x * 8;
    float sum = 0.f;
    if (col < h) {
      float a[8], b[8];
      unpack8<__half>(*reinterpret_cast<const uint4*>(dout + row * h + col), a);
      unpack8<__half>(*reinterpret_cast<const uint4*>(out + row * h + col), b);
#pragma unroll
      for (int j = 0; j < 8; ++j) sum = fmaf(a[j], b[j], sum);
    }
#pragma unroll
    for (int o = kLanesPerHead / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (col < h && (threadIdx.x & (kLanesPerHead - 1)) == 0) {
      const int head = col / HD;
      const int chunk = row >= c ? 1 : 0;
      if (dbg_ok(row - chunk * c < c, nullptr))
        delta[(static_cast<int64_t>(head) * 2 + chunk) * c_pad + (row - chunk * c)] = scale * sum;
    }
  }
}

}  // namespace tsp
