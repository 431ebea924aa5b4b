// attn_sm100.cuh - causal flash attention of one TSP rank's queries against the
// all-gathered full-sequence K/V, for sm_100a tensor cores.
//
// What it computes (TSP news item, zubnet.ai, paragraph 2: each rank applies
// the attention shards to its own tokens against the K/V all-gathered under
// the zigzag partition): for every local query row i at global position
// p(i) and every head j,
//     A[i, j] = softmax_k<=p(i) (scale * q_ij . k_kj) . v_kj.
// The rank's rows are two chunks (r and 2D-1-r) of c tokens.  A query tile
// of 128 rows lies inside one chunk, so its positions are contiguous and it
// needs key tiles 0 .. (last position)/128 only: key tiles past the chunk's
// end are never loaded (chunk skipping).  Only tiles that reach past the
// tile's first position apply the causal mask.
//
// Work item = (query tile, head).  Items are handed out through an atomic
// counter in the order: heavy chunk (2D-1-r) first, head-major, descending
// position; then the light chunk.  Heavy items come first so that the
// greedy queue finishes balanced (longest-processing-time order), and
// head-major order makes the ~148 concurrent items stream the same head's
// K/V so each tile is read from HBM about once and served from L2.
//
// Roles (320 threads, one CTA per SM, persistent):
//   warp 0     work queue + TMA producer (Q tile, K ring, V ring)
//   warp 1     TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-9  softmax / correction / epilogue.  Warp w reads TMEM lanes
//              32*(w%4).. (its 32 query rows) and owns half (w-2)/4 of the
//              128 key columns of each score tile and of the d output
//              columns: two warps per row quarter, so each SM sub-partition
//              interleaves two softmax warps.  Both compute the full row
//              maximum (the lazy rescale must agree); each exponentiates and
//              stores only its 64 columns; the two partial row sums are
//              added once per work item through shared memory.
// Tensor memory (512 columns): S0 | S1 (128 fp32 columns each, double
// buffered scores), O (d fp32 columns), P0 | P1 (64 columns each: 128 fp16
// probabilities packed in pairs, the A operand of O += P V).  Q, K, V and
// the output are fp16; scores, the softmax statistics and O are fp32.
// Online softmax in base 2 with a lazily updated row maximum: the running
// output is rescaled only when the maximum grows by more than 2^8, which is
// exact (the final division by the row sum cancels the common factor).
#pragma once
#include "gemm_sm100.cuh"
#include "ptx.cuh"

namespace tsp {

constexpr int kAttnSoftmaxWarps = 8;
constexpr int kAttnThreads = 64 + 32 * kAttnSoftmaxWarps;
constexpr int kAttnBM = 128;
constexpr int kAttnBN = 128;

struct __align__(64) AttnParams {
  CUtensorMap map_q;  // Q [L, h] fp16, box {64, 128}
  CUtensorMap map_k;  // K [T, h] fp16, box {64, 128}
  CUtensorMap map_v;  // V [T, h] fp16, box {64, 128}
  __half* out;        // A [L, h] fp16
  int64_t ldo;        // h
  int c;              // chunk length
  int rank, D, H;
  int nqt;            // query tiles per chunk
  int n_items;        // 2 * nqt * H
  float scale_log2;   // softmax scale * log2(e)
  int* counter;       // work queue head (zeroed before launch)
  int* status;
  uint64_t timeout_ns;
};

template <int HD>
struct AttnShape {
  static constexpr int kQBytes = kAttnBM * HD * 2;
  static constexpr int kKVBytes = kAttnBN * HD * 2;
  static constexpr int kStages = (HD == 128) ? 3 : 4;
  static constexpr int kBarBytes = 512 + 1024;  // barriers + row-sum exchange
  static constexpr int kSmemBytes = kQBytes + 2 * kStages * kKVBytes + kBarBytes + 1024;
  static constexpr uint32_t kColS = 0, kColO = 256, kColP = 384;
};

struct AttnItem {
  int head, m0, p0, nvalid, nkv;
};

__device__ __forceinline__ AttnItem attn_decode(const AttnParams& p, int it) {
  const int per_chunk = p.nqt * p.H;
  const int heavy = it < per_chunk;
  const int ii = heavy ? it : it - per_chunk;
  AttnItem w;
  w.head = ii / p.nqt;
  const int t = p.nqt - 1 - (ii % p.nqt);
  const int chunk_local = heavy ? 1 : 0;
  const int gchunk = heavy ? (2 * p.D - 1 - p.rank) : p.rank;
  w.m0 = chunk_local * p.c + t * kAttnBM;
  w.p0 = gchunk * p.c + t * kAttnBM;
  w.nvalid = min(kAttnBM, p.c - t * kAttnBM);
  w.nkv = (w.p0 + w.nvalid - 1) / kAttnBN + 1;
  return w;
}

// Every lane of the warp waits, then the warp agrees: if any lane gave up
// (abort or timeout) the whole warp leaves together, so the .sync.aligned
// tensor-memory instructions that follow are never reached by half a warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const bool ok = mbar_wait(bar, parity, ctl);
  return __all_sync(0xffffffffu, ok);
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_tcgen05(const __grid_constant__ AttnParams p) {
  using S = AttnShape<HD>;
  constexpr int STAGES = S::kStages;
  constexpr int NB = HD / 64;  // 64-column (128-byte) boxes per row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + S::kQBytes;
  uint8_t* sV = sK + STAGES * S::kKVBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + STAGES * S::kKVBytes);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* k_full = bars + 2;
  uint64_t* k_empty = k_full + STAGES;
  uint64_t* v_full = k_empty + STAGES;
  uint64_t* v_empty = v_full + STAGES;
  uint64_t* s_full = v_empty + STAGES;  // [2]
  uint64_t* s_free = s_full + 2;        // [2]
  uint64_t* p_full = s_free + 2;        // [2]
  uint64_t* o_done = p_full + 2;        // [2], by PV index parity
  uint64_t* o_free = o_done + 2;
  uint64_t* it_full = o_free + 1;       // [2]
  uint64_t* it_empty = it_full + 2;     // [2]
  uint64_t* drain = it_empty + 2;
  uint64_t* sum_bar = drain + 1;        // [4], one per row quarter: both halves' row sums written
  int* it_slot = reinterpret_cast<int*>(sum_bar + 4);  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(it_slot + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* red_sum = reinterpret_cast<float*>(bars) + 128;  // [2 halves][128 rows], after 512 B of barriers

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_free[b], kAttnSoftmaxWarps);
      mbar_init(&p_full[b], kAttnSoftmaxWarps);
      mbar_init(&o_done[b], 1);
      mbar_init(&it_full[b], 1);
      mbar_init(&it_empty[b], 1 + kAttnSoftmaxWarps);
    }
    mbar_init(o_free, kAttnSoftmaxWarps);
    mbar_init(drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&sum_bar[q], 2);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      tma_prefetch_desc(&p.map_q);
      tma_prefetch_desc(&p.map_k);
      tma_prefetch_desc(&p.map_v);
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph = 0;
      uint32_t kused = 0, kpar = 0, vused = 0, vpar = 0, qused = 0, qpar = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait(&it_empty[slot], ((n >> 1) & 1) ^ 1, ctl)) break;
        int it = atomicAdd(p.counter, 1);
        if (it >= p.n_items) it = -1;
        it_slot[slot] = it;
        mbar_arrive(&it_full[slot]);
        if (it < 0) break;
        const AttnItem w = attn_decode(p, it);
        const int col0 = w.head * HD;
        if (!mbar_wait(q_empty, qph ^ 1, ctl)) break;
        mbar_arrive_expect_tx(q_full, S::kQBytes);
#pragma unroll
        for (int b = 0; b < NB; ++b) tma_load_2d(sQ + b * 16384, &p.map_q, q_full, col0 + 64 * b, w.m0);
        qused = 1;
        qpar = qph;
        qph ^= 1;
        for (int kt = 0; kt < w.nkv; ++kt) {
          if (!mbar_wait(&k_empty[ks], kph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[ks], S::kKVBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sK + ks * S::kKVBytes + b * 16384, &p.map_k, &k_full[ks], col0 + 64 * b, kt * kAttnBN);
          kused |= 1u << ks;
          kpar = (kpar & ~(1u << ks)) | (kph << ks);
          if (++ks == STAGES) { ks = 0; kph ^= 1; }
          if (!mbar_wait(&v_empty[vs], vph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[vs], S::kKVBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sV + vs * S::kKVBytes + b * 16384, &p.map_v, &v_full[vs], col0 + 64 * b, kt * kAttnBN);
          vused |= 1u << vs;
          vpar = (vpar & ~(1u << vs)) | (vph << vs);
          if (++vs == STAGES) { vs = 0; vph ^= 1; }
        }
      }
      if (qused) mbar_drain(q_full, qpar, p.timeout_ns);
      for (int s = 0; s < STAGES; ++s) {
        if (kused & (1u << s)) mbar_drain(&k_full[s], (kpar >> s) & 1, p.timeout_ns);
        if (vused & (1u << s)) mbar_drain(&v_full[s], (vpar >> s) & 1, p.timeout_ns);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_f32acc(kAttnBM, kAttnBN, 0, 0, kFmtF16);
      constexpr uint32_t idesc_o = idesc_f32acc(kAttnBM, HD, 0, 1, kFmtF16);
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph = 0;
      uint32_t g = 0;      // global score-tile counter (S/P buffer = g & 1)
      int items = 0;
      bool ok = true;
      // S_gg = Q K^T into S buffer gg & 1; last = the item's final score tile
      auto issue_s = [&](uint32_t gg, bool last) -> bool {
        const int sb = gg & 1;
        if (!mbar_wait(&s_free[sb], ((gg >> 1) & 1) ^ 1, ctl)) return false;
        if (!mbar_wait(&k_full[ks], kph, ctl)) return false;
        tc_fence_after();
        const uint32_t q0 = smem_u32(sQ);
        const uint32_t k0 = smem_u32(sK + ks * S::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < HD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + S::kColS + sb * 128, smem_desc_sw128(q0 + off, 16, 1024),
                 smem_desc_sw128(k0 + off, 16, 1024), idesc_s, kk != 0);
        }
        mma_commit(&k_empty[ks]);
        mma_commit(&s_full[sb]);
        if (last) mma_commit(q_empty);
        if (++ks == STAGES) { ks = 0; kph ^= 1; }
        return true;
      };
      // O += P_gg V; first = first PV of the item (overwrites O)
      auto issue_pv = [&](uint32_t gg, bool first) -> bool {
        const int pb = gg & 1;
        if (first && !mbar_wait(o_free, (items & 1) ^ 1, ctl)) return false;
        if (!mbar_wait(&p_full[pb], (gg >> 1) & 1, ctl)) return false;
        if (!mbar_wait(&v_full[vs], vph, ctl)) return false;
        tc_fence_after();
        const uint32_t v0 = smem_u32(sV + vs * S::kKVBytes);
#pragma unroll
        for (int kk = 0; kk < kAttnBN / 16; ++kk) {
          const uint64_t bd = smem_desc_sw128(v0 + kk * 2048, 16384, 1024);
          mma_ts(tmem + S::kColO, tmem + S::kColP + pb * 64 + kk * 8, bd, idesc_o, !(first && kk == 0));
        }
        mma_commit(&v_empty[vs]);
        mma_commit(&o_done[gg & 1]);
        if (++vs == STAGES) { vs = 0; vph ^= 1; }
        return true;
      };
      // Issue order per item: S_0, S_1, then for each tile j: S_{j+2}, PV_j.
      // Scores run two tiles ahead of the softmax, so the tensor core computes
      // S_{j+2} while the softmax works on tile j and PV_j follows as soon as
      // P_j is written.
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait(&it_full[slot], (n >> 1) & 1, ctl)) break;
        const int it = it_slot[slot];
        mbar_arrive(&it_empty[slot]);
        if (it < 0) break;
        const AttnItem w = attn_decode(p, it);
        if (!mbar_wait(q_full, qph, ctl)) break;
        qph ^= 1;
        const int pre = w.nkv < 2 ? w.nkv : 2;
        for (int t = 0; ok && t < pre; ++t) ok = issue_s(g + t, t == w.nkv - 1);
        for (int kt = 0; ok && kt < w.nkv; ++kt) {
          if (kt + 2 < w.nkv) ok = issue_s(g + kt + 2, kt + 2 == w.nkv - 1);
          if (ok) ok = issue_pv(g + kt, kt == 0);
        }
        if (!ok) break;
        g += w.nkv;
        ++items;
      }
      mma_commit(drain);
      mbar_drain(drain, 0, p.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    constexpr int HALF_D = HD / 2;
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = p.scale_log2;
    uint32_t g = 0;
    uint32_t done_items = 0;
    for (int n = 0;; ++n) {
      const int slot = n & 1;
      if (!warp_wait(&it_full[slot], (n >> 1) & 1, ctl)) break;
      const int it = it_slot[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&it_empty[slot]);
      if (it < 0) break;
      const AttnItem w = attn_decode(p, it);
      const int qpos = w.p0 + row;
      const bool row_valid = row < w.nvalid;
      float m_used = -INFINITY;
      float l = 0.f;  // this warp's half of the row sum
      bool ok = true;
      for (int kt = 0; kt < w.nkv; ++kt, ++g) {
        const int sb = g & 1;
        if (!warp_wait(&s_full[sb], (g >> 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        // own[]: this warp's 64 key columns; oth[]: the partner warp's 64
        uint32_t own[64], oth[64];
        {
          const uint32_t sbase = tmem + lane_off + S::kColS + sb * 128;
          tmem_ld32p(sbase + half * 64, &own[0]);
          tmem_ld32p(sbase + half * 64 + 32, &own[32]);
          tmem_ld32p(sbase + (1 - half) * 64, &oth[0]);
          tmem_ld32p(sbase + (1 - half) * 64 + 32, &oth[32]);
          tmem_ld_wait();
          reg_fence32(&own[0]);
          reg_fence32(&own[32]);
          reg_fence32(&oth[0]);
          reg_fence32(&oth[32]);
        }
        float* so = reinterpret_cast<float*>(own);
        float* st = reinterpret_cast<float*>(oth);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[sb]);
        const int kbase = kt * kAttnBN;
        if (kbase + kAttnBN - 1 > w.p0) {
          const int ko = kbase + half * 64, kx = kbase + (1 - half) * 64;
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            if (ko + i > qpos) so[i] = -INFINITY;
            if (kx + i > qpos) st[i] = -INFINITY;
          }
        }
        float mx;
        {  // full row maximum (both warps of the row quarter get the same value)
          float m8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) m8[k] = fmaxf(so[k], st[k]);
#pragma unroll
          for (int i = 8; i < 64; i += 8)
#pragma unroll
            for (int k = 0; k < 8; ++k) m8[k] = fmax3(m8[k], so[i + k], st[i + k]);
          mx = fmax3(fmax3(m8[0], m8[1], m8[2]), fmax3(m8[3], m8[4], m8[5]), fmaxf(m8[6], m8[7]));
        }
        const float m_new = fmaxf(m_used, mx * sl2);
        const bool need = m_new > m_used + 8.0f;
        if (kt > 0 && __any_sync(0xffffffffu, need)) {
          // the previous P V product must land before O is rescaled
          if (!warp_wait(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, ctl)) { ok = false; break; }
          tc_fence_after();
          const float f = need ? ex2_approx(m_used - m_new) : 1.0f;
#pragma unroll
          for (int j = 0; j < HALF_D / 32; ++j) {
            uint32_t r[32];
            const uint32_t a = tmem + lane_off + S::kColO + half * HALF_D + j * 32;
            tmem_ld32(a, r);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
            tmem_st32(a, r);
          }
          if (need) l *= f;
        }
        if (need) m_used = m_new;
        // P buffer g & 1 was last read by PV_{g-2}, which the tensor core may
        // still be running (scores are issued ahead of it)
        if (g >= 2 && !warp_wait(&o_done[g & 1], ((g - 2) >> 1) & 1, ctl)) { ok = false; break; }
        {
          // this warp's 64 probabilities 2^(s*scale*log2e - m) as 32 pairs in
          // f32x2 arithmetic; one pair in four on the FMA pipes (polynomial),
          // the rest on MUFU; the partial row sum in two packed accumulators
          const int pb = g & 1;
          const float neg_m = -m_used;
          const float2 sl2v = make_float2(sl2, sl2), negm = make_float2(neg_m, neg_m);
          float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float2 x = ffma2(make_float2(so[2 * i], so[2 * i + 1]), sl2v, negm);
            float2 pr;
            if ((i & 3) == 3) {
              pr = exp2_poly2(x);
            } else {
              pr.x = ex2_approx(x.x);
              pr.y = ex2_approx(x.y);
            }
            if (i & 1) lb = fadd2(lb, pr); else la = fadd2(la, pr);
            r[i] = pack_half2(pr.x, pr.y);
          }
          tmem_st32(tmem + lane_off + S::kColP + pb * 64 + half * 32, r);
          const float2 lab = fadd2(la, lb);
          l += lab.x + lab.y;
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[pb]);
        }
      }
      if (!ok) break;
      // epilogue: row sum from both halves, then O / l -> fp16 -> A[m0 + row, head]
      const uint32_t gl = g - 1;
      if (!warp_wait(&o_done[gl & 1], (gl >> 1) & 1, ctl)) break;
      tc_fence_after();
      red_sum[half * 128 + row] = l;
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sum_bar[quarter]);
      if (!warp_wait(&sum_bar[quarter], done_items & 1, ctl)) break;
      ++done_items;
      const float inv = 1.0f / (red_sum[row] + red_sum[128 + row]);
      __half* dst = p.out + static_cast<int64_t>(w.m0 + row) * p.ldo + w.head * HD + half * HALF_D;
#pragma unroll
      for (int j = 0; j < HALF_D / 32; ++j) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + S::kColO + half * HALF_D + j * 32, r);
        tmem_ld_wait();
        if (row_valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + j * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(pack_half2(__uint_as_float(r[8 * i]) * inv, __uint_as_float(r[8 * i + 1]) * inv),
                               pack_half2(__uint_as_float(r[8 * i + 2]) * inv, __uint_as_float(r[8 * i + 3]) * inv),
                               pack_half2(__uint_as_float(r[8 * i + 4]) * inv, __uint_as_float(r[8 * i + 5]) * inv),
                               pack_half2(__uint_as_float(r[8 * i + 6]) * inv, __uint_as_float(r[8 * i + 7]) * inv));
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tsp
