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
// Work item = (pair of adjacent query tiles of one chunk, head).  Both tiles
// of a pair stream the same K/V tiles, so each K/V tile brought into shared
// memory feeds two 128-row score tiles.  Items are handed out through an
// atomic counter in the order: heavy chunk (2D-1-r) first, head-major,
// descending position; then the light chunk.  Heavy items first makes the
// greedy queue finish balanced (longest-processing-time order); head-major
// order makes the ~148 concurrent items stream the same head's K/V, so each
// K/V tile is read from HBM about once and then served from L2.
//
// Roles (384 threads = three warpgroups, one CTA per SM, persistent):
//   warp 0      work queue + TMA producer (Q_A, Q_B, K ring, V ring)
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2-3   idle (they complete the first warpgroup)
//   warps 4-7   softmax, correction and epilogue of query tile A (thread = row)
//   warps 8-11  the same for query tile B
// Each SM sub-partition runs one warp of each warpgroup.  The registers are
// re-split at the start (setmaxnreg): the first warpgroup drops to
// kAttnLowRegs per thread and the two softmax warpgroups rise to
// kAttnHighRegs (128 x 56 + 256 x 224 = 384 x 168, the launch allocation,
// which the launcher checks).  At the 168 of a uniform split the softmax
// spilled, and reloading the spills cost 6% of the kernel's time.
// Tensor memory (512 columns): [S | P_A | P_B | O_A | O_B] = 128 + 64 + 64 +
// 128 + 128.  The score buffer S is shared by the two query tiles and used in
// turn: S_A(j), S_B(j), S_A(j+1), ...  A softmax warp reads its whole score
// tile into registers and at once hands S back to the issuer, which computes
// the other tile's scores while the softmax turns its registers into fp16
// probabilities P in the tile's own P region.  The tensor core is fed in the
// order S_A(j+1) PV_A(j) S_B(j+1) PV_B(j) ..., so the next scores of a tile
// never wait for its PV, and a softmax warp never waits for the tensor core
// except for its next score tile.  P_x is rewritten only after the PV that
// read it has finished (one commit per PV).
// Online softmax in base 2 with a lazily moved offset: a row subtracts the
// maximum of its first key tile from every later score, with no maximum pass
// over the later tiles.  Any common offset is exact (the final division by
// the row sum cancels it); the offset only has to keep every probability
// inside fp16's range.  A tile's fp32 row sum bounds its largest probability
// (every exponential is a MUFU ex2, which gives +inf past fp32's range): a
// sum above 2^15 sends that row's tile down a rare path, which recomputes the
// row's 128 scores from Q and K in global memory on the CUDA cores, moves the
// offset to their maximum, redoes the probabilities and rescales O before the
// next PV.
// Q, K, V, P and the output are fp16; scores, softmax statistics and O are
// fp32.
#pragma once
#include "gemm_sm100.cuh"
#include "ptx.cuh"

namespace tsp {

constexpr int kAttnThreads = 384;
constexpr int kAttnLaunchRegs = 168;  // per thread at launch: 65536 / 384, rounded down to 8
constexpr int kAttnLowRegs = 56;      // warps 0-3 after the re-split
constexpr int kAttnHighRegs = 224;    // the softmax warpgroups after the re-split
static_assert(128 * kAttnLowRegs + 256 * kAttnHighRegs <= kAttnThreads * kAttnLaunchRegs, "register split");
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
  int npairs;         // query-tile pairs per chunk, ceil(nqt / 2)
  int n_items;        // 2 * npairs * H
  float scale_log2;   // softmax scale * log2(e)
  int* counter;       // work queue head (zeroed before launch)
  int* status;
  uint64_t timeout_ns;
  // Optional stash for the backward: per row and head the log-sum-exp of the
  // row's scaled scores in log2 units, lse2 = log2 sum_k 2^(s_k * scale *
  // log2 e), so that P = 2^(s * scale * log2 e - lse2).  Layout [H][2][c_pad]
  // fp32: head, local chunk, row within the chunk (c_pad = c rounded up to a
  // multiple of 128, so every 128-row tile of a chunk starts 512-byte aligned).
  float* lse;
  int c_pad;
  // Q and K again as plain row-major arrays (row stride ldqk elements), read
  // only on the rare path that recomputes a score row on the CUDA cores.
  const __half* q;
  const __half* k;
  int64_t ldqk;
};

template <int HD>
struct AttnShape {
  static constexpr int kQBytes = kAttnBM * HD * 2;
  static constexpr int kKVBytes = kAttnBN * HD * 2;
  static constexpr int kKStages = (HD == 128) ? 3 : 4;
  static constexpr int kVStages = (HD == 128) ? 2 : 4;
  static constexpr int kBarBytes = 512;
  static constexpr int kSmemBytes = 2 * kQBytes + (kKStages + kVStages) * kKVBytes + kBarBytes + 1024;
};

struct AttnTile {
  int m0, p0, nvalid, nkv;  // nkv == 0: the tile does not exist
};
struct AttnItem {
  int head;
  AttnTile t[2];
};

__device__ __forceinline__ AttnItem attn_decode(const AttnParams& p, int it) {
  const int per_chunk = p.npairs * p.H;
  const int heavy = it < per_chunk;
  const int ii = heavy ? it : it - per_chunk;
  AttnItem w;
  w.head = ii / p.npairs;
  const int pr = p.npairs - 1 - (ii % p.npairs);
  const int gchunk = heavy ? (2 * p.D - 1 - p.rank) : p.rank;
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int t = 2 * pr + x;
    if (t < p.nqt) {
      w.t[x].m0 = heavy * p.c + t * kAttnBM;
      w.t[x].p0 = gchunk * p.c + t * kAttnBM;
      w.t[x].nvalid = min(kAttnBM, p.c - t * kAttnBM);
      w.t[x].nkv = (w.t[x].p0 + w.t[x].nvalid - 1) / kAttnBN + 1;
    } else {
      w.t[x].m0 = w.t[x].p0 = w.t[x].nvalid = w.t[x].nkv = 0;
    }
  }
  return w;
}

// Maximum of a 128-entry row (three-input maxima in four chains).
__device__ __forceinline__ float attn_row_max(const float* sv) {
  float m4[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) m4[k] = fmaxf(sv[k], sv[k + 4]);
#pragma unroll
  for (int i = 8; i < 128; i += 8)
#pragma unroll
    for (int k = 0; k < 4; ++k) m4[k] = fmax3(m4[k], sv[i + k], sv[i + k + 4]);
  return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
}

// P = 2^(s * sl2 - m) for a 128-entry score row as 64 fp16 pairs (MUFU
// ex2: +inf past fp32's range, +0 below it); returns the row sum of the fp32
// values.
__device__ __forceinline__ float attn_exp_pack(const float* sv, float sl2, float m, uint32_t* P) {
  float2 la = make_float2(0.f, 0.f), lb = make_float2(0.f, 0.f);
  const float2 sl2v = make_float2(sl2, sl2), negm = make_float2(-m, -m);
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float2 xv = ffma2(make_float2(sv[2 * i], sv[2 * i + 1]), sl2v, negm);
    float2 pr;
    pr.x = ex2_approx(xv.x);
    pr.y = ex2_approx(xv.y);
    if (i & 1) lb = fadd2(lb, pr); else la = fadd2(la, pr);
    P[i] = pack_half2(pr.x, pr.y);
  }
  const float2 lab = fadd2(la, lb);
  return lab.x + lab.y;
}

// One query row's scores against keys kbase .. kbase+127 of one head, in
// fp32 on the CUDA cores (keys past the row's position get -inf; a row past
// the tile's valid rows gets zeros).  Only the rare path uses it.
template <int HD>
__device__ __forceinline__ void attn_scores_from_global(const AttnParams& p, int head, int qrow, int kbase, int qpos,
                                                        bool row_valid, float* sv) {
  // (the debug build checks the row, the head and the row's position, which
  // bounds every key read below it)
  const bool ok = row_valid && dbg_ok(qrow < 2 * p.c && qpos < 2 * p.D * p.c && (head + 1) * HD <= p.ldqk, p.status);
  const uint4* qr = reinterpret_cast<const uint4*>(p.q + static_cast<int64_t>(qrow) * p.ldqk + head * HD);
#pragma unroll 1
  for (int i = 0; i < 128; ++i) {
    const int key = kbase + i;
    float acc = row_valid ? -INFINITY : 0.f;
    if (ok && key <= qpos) {
      const uint4* kr = reinterpret_cast<const uint4*>(p.k + static_cast<int64_t>(key) * p.ldqk + head * HD);
      acc = 0.f;
#pragma unroll 1
      for (int d = 0; d < HD / 8; ++d) {
        const uint4 a = qr[d], b = kr[d];
        const __half2* ah = reinterpret_cast<const __half2*>(&a);
        const __half2* bh = reinterpret_cast<const __half2*>(&b);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 af = __half22float2(ah[e]), bf = __half22float2(bh[e]);
          acc = fmaf(af.x, bf.x, acc);
          acc = fmaf(af.y, bf.y, acc);
        }
      }
    }
    sv[i] = acc;
  }
}

// Every lane of the warp waits, then the warp agrees: if any lane gave up
// (abort or timeout) the whole warp leaves together, so the .sync.aligned
// tensor-memory instructions that follow are never reached by half a warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& ctl) {
  const bool ok = mbar_wait_inl(bar, parity, ctl);
  return __all_sync(0xffffffffu, ok);
}

template <int HD>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_tcgen05(const __grid_constant__ AttnParams p) {
  using S = AttnShape<HD>;
  constexpr int KST = S::kKStages;
  constexpr int VST = S::kVStages;
  constexpr int NB = HD / 64;  // 64-column (128-byte) boxes per row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // [2][kQBytes]
  uint8_t* sK = sQ + 2 * S::kQBytes;        // [KST][kKVBytes]
  uint8_t* sV = sK + KST * S::kKVBytes;     // [VST][kKVBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + VST * S::kKVBytes);
  uint64_t* q_full = bars;                  // [2]
  uint64_t* q_empty = q_full + 2;           // [2]
  uint64_t* k_full = q_empty + 2;           // [KST]
  uint64_t* k_empty = k_full + KST;         // [KST]
  uint64_t* v_full = k_empty + KST;         // [VST]
  uint64_t* v_empty = v_full + VST;         // [VST]
  uint64_t* s_full = v_empty + VST;         // [2] S holds the scores of query tile x
  uint64_t* p_full = s_full + 2;            // [2] probabilities of tile x written
  uint64_t* o_full = p_full + 2;            // [2] last PV of tile x done
  uint64_t* o_free = o_full + 2;            // [2] epilogue of tile x has read O
  uint64_t* pv_done = o_free + 2;           // [2] a PV of tile x (not its last) done
  uint64_t* s_free = pv_done + 2;           // the scores in S have been read
  uint64_t* it_full = s_free + 1;           // [2]
  uint64_t* it_empty = it_full + 2;         // [2]
  uint64_t* drain = it_empty + 2;
  int* it_slot = reinterpret_cast<int*>(drain + 1);  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(it_slot + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&o_full[x], 1);
      mbar_init(&o_free[x], 4);
      mbar_init(&pv_done[x], 1);
      mbar_init(&it_full[x], 1);
      mbar_init(&it_empty[x], 9);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(s_free, 4);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl ctl{abort_flag, p.status, p.timeout_ns};

  if (warp < 4) {
    __syncwarp();
    regs_dec<kAttnLowRegs>();
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (elect_one()) {
      tma_prefetch_desc(&p.map_q);
      tma_prefetch_desc(&p.map_k);
      tma_prefetch_desc(&p.map_v);
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph[2] = {0, 0};
      uint32_t kused = 0, kpar = 0, vused = 0, vpar = 0, qused = 0, qpar = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait_inl(&it_empty[slot], ((n >> 1) & 1) ^ 1, ctl)) break;
        int it = atomicAdd(p.counter, 1);
        if (it >= p.n_items) it = -1;
        it_slot[slot] = it;
        mbar_arrive(&it_full[slot]);
        if (it < 0) break;
        const AttnItem w = attn_decode(p, it);
        const int col0 = w.head * HD;
        for (int x = 0; ok && x < 2; ++x) {
          if (w.t[x].nkv == 0) continue;
          if (!mbar_wait_inl(&q_empty[x], qph[x] ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[x], S::kQBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sQ + x * S::kQBytes + b * 16384, &p.map_q, &q_full[x], col0 + 64 * b, w.t[x].m0);
          qused |= 1u << x;
          qpar = (qpar & ~(1u << x)) | (qph[x] << x);
          qph[x] ^= 1;
        }
        const int nkv = max(w.t[0].nkv, w.t[1].nkv);
        for (int kt = 0; ok && kt < nkv; ++kt) {
          if (!mbar_wait_inl(&k_empty[ks], kph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&k_full[ks], S::kKVBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sK + ks * S::kKVBytes + b * 16384, &p.map_k, &k_full[ks], col0 + 64 * b, kt * kAttnBN);
          kused |= 1u << ks;
          kpar = (kpar & ~(1u << ks)) | (kph << ks);
          if (++ks == KST) { ks = 0; kph ^= 1; }
          if (!mbar_wait_inl(&v_empty[vs], vph ^ 1, ctl)) { ok = false; break; }
          mbar_arrive_expect_tx(&v_full[vs], S::kKVBytes);
#pragma unroll
          for (int b = 0; b < NB; ++b)
            tma_load_2d(sV + vs * S::kKVBytes + b * 16384, &p.map_v, &v_full[vs], col0 + 64 * b, kt * kAttnBN);
          vused |= 1u << vs;
          vpar = (vpar & ~(1u << vs)) | (vph << vs);
          if (++vs == VST) { vs = 0; vph ^= 1; }
        }
      }
      for (int x = 0; x < 2; ++x)
        if (qused & (1u << x)) mbar_drain(&q_full[x], (qpar >> x) & 1, p.timeout_ns);
      for (int s = 0; s < KST; ++s)
        if (kused & (1u << s)) mbar_drain(&k_full[s], (kpar >> s) & 1, p.timeout_ns);
      for (int s = 0; s < VST; ++s)
        if (vused & (1u << s)) mbar_drain(&v_full[s], (vpar >> s) & 1, p.timeout_ns);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_s = idesc_f32acc(kAttnBM, kAttnBN, 0, 0, kFmtF16);
      constexpr uint32_t idesc_o = idesc_f32acc(kAttnBM, HD, 0, 1, kFmtF16);
      int ks = 0, vs = 0;
      uint32_t kph = 0, vph = 0, qph[2] = {0, 0};
      uint32_t pcnt[2] = {0, 0};  // probability tiles consumed, per query-tile slot
      uint32_t icnt[2] = {0, 0};  // items finished, per query-tile slot
      uint32_t scnt = 0;          // score tiles issued (S is reused after each is read)
      bool ok = true;
      // Shared-memory descriptors of every Q and K/V stage, built once; an MMA
      // group then only adds immediate offsets (see mma_ss_x8 / mma_ts_x8).
      const uint64_t qdesc0 = smem_desc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t vdesc0 = smem_desc_sw128(smem_u32(sV), 16384, 1024);
      auto qdesc = [&](int x) { return qdesc0 + static_cast<uint64_t>(x * (S::kQBytes >> 4)); };
      auto kdesc = [&]() { return kdesc0 + static_cast<uint64_t>(ks * (S::kKVBytes >> 4)); };
      auto vdesc = [&]() { return vdesc0 + static_cast<uint64_t>(vs * (S::kKVBytes >> 4)); };
      // S_x = Q_x K^T for the K tile in slot ks (K = head_dim in 16-column steps:
      // +32 bytes inside a 128-byte swizzle row, +16 KiB to the next 64 columns)
      auto issue_s = [&](int x, bool last_s) -> bool {
        if (scnt > 0 && !mbar_wait_inl(s_free, (scnt - 1) & 1, ctl)) return false;
        ++scnt;
        tc_fence_after();
        if constexpr (HD == 128) {
          mma_ss_x8<0, 2, 4, 6, 1024, 1026, 1028, 1030>(tmem, qdesc(x), kdesc(), idesc_s, 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < HD / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            mma_ss(tmem, qdesc(x) + off, kdesc() + off, idesc_s, kk != 0);
          }
        }
        mma_commit(&s_full[x]);
        if (last_s) mma_commit(&q_empty[x]);
        return true;
      };
      // O_x += P_x V for the V tile in slot vs (K = 128 keys in 16-key steps:
      // P advances 8 TMEM columns, V 2 KiB = 128 units)
      auto issue_pv = [&](int x, bool first, bool last) -> bool {
        if (first && !mbar_wait_inl(&o_free[x], (icnt[x] & 1) ^ 1, ctl)) return false;
        if (!mbar_wait_inl(&p_full[x], pcnt[x] & 1, ctl)) return false;
        ++pcnt[x];
        tc_fence_after();
        mma_ts_x8<128>(tmem + 256 + x * 128, tmem + 128 + x * 64, vdesc(), idesc_o, first ? 0u : 1u);
        mma_commit(last ? &o_full[x] : &pv_done[x]);
        return true;
      };
      auto wait_k = [&]() -> bool {
        if (!mbar_wait_inl(&k_full[ks], kph, ctl)) return false;
        tc_fence_after();
        return true;
      };
      auto release_k = [&]() {
        mma_commit(&k_empty[ks]);
        if (++ks == KST) { ks = 0; kph ^= 1; }
      };
      for (int n = 0; ok; ++n) {
        const int slot = n & 1;
        if (!mbar_wait_inl(&it_full[slot], (n >> 1) & 1, ctl)) break;
        const int it = it_slot[slot];
        mbar_arrive(&it_empty[slot]);
        if (it < 0) break;
        const AttnItem w = attn_decode(p, it);
        const int na = w.t[0].nkv, nb = w.t[1].nkv;
        const int nkv = max(na, nb);
        for (int x = 0; ok && x < 2; ++x) {
          if (w.t[x].nkv == 0) continue;
          ok = mbar_wait_inl(&q_full[x], qph[x], ctl);
          qph[x] ^= 1;
        }
        if (!ok) break;
        tc_fence_after();
        // scores of K tile 0 for both query tiles
        if (!wait_k()) break;
        if (na > 0 && !issue_s(0, na == 1)) break;
        if (nb > 0 && !issue_s(1, nb == 1)) break;
        release_k();
        // per key tile: S_A(kt+1) PV_A(kt) S_B(kt+1) PV_B(kt)
        for (int kt = 0; ok && kt < nkv; ++kt) {
          if (!mbar_wait_inl(&v_full[vs], vph, ctl)) { ok = false; break; }
          bool k_waited = false;
          if (kt < na) {
            if (kt + 1 < na) {
              if (!wait_k()) { ok = false; break; }
              k_waited = true;
              if (!issue_s(0, kt + 1 == na - 1)) { ok = false; break; }
            }
            if (!issue_pv(0, kt == 0, kt == na - 1)) { ok = false; break; }
          }
          if (kt < nb) {
            if (kt + 1 < nb) {
              if (!k_waited) {
                if (!wait_k()) { ok = false; break; }
                k_waited = true;
              }
              if (!issue_s(1, kt + 1 == nb - 1)) { ok = false; break; }
            }
            if (!issue_pv(1, kt == 0, kt == nb - 1)) { ok = false; break; }
          }
          if (k_waited) release_k();
          mma_commit(&v_empty[vs]);
          if (++vs == VST) { vs = 0; vph ^= 1; }
        }
        if (!ok) break;
        for (int x = 0; x < 2; ++x)
          if (w.t[x].nkv > 0) ++icnt[x];
      }
      mma_commit(drain);
      mbar_drain(drain, 0, p.timeout_ns);
    }
  }
  } else {
    // ---------------------------------------------------------------- softmax
    __syncwarp();
    regs_inc<kAttnHighRegs>();
    const int x = (warp - 4) >> 2;     // query tile of this warp group
    const int quarter = warp & 3;      // TMEM lane quarter = rows 32*quarter ..
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_off;                  // S (shared by both tiles)
    const uint32_t t_p = tmem + lane_off + 128 + x * 64;   // P of this tile
    const uint32_t t_o = tmem + lane_off + 256 + x * 128;  // O of this tile
    const float sl2 = p.scale_log2;
    uint32_t scnt = 0, icnt = 0, pvcnt = 0;
    for (int n = 0;; ++n) {
      const int slot = n & 1;
      if (!warp_wait(&it_full[slot], (n >> 1) & 1, ctl)) break;
      const int it = it_slot[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&it_empty[slot]);
      if (it < 0) break;
      // Only the key-loop's own values stay live across it (registers are
      // tight here): the rare path and the epilogue decode the item again.
      const int nkv_x = attn_decode(p, it).t[x].nkv;
      if (nkv_x == 0) continue;
      const int p0_x = attn_decode(p, it).t[x].p0;
      const int qpos = p0_x + row;
      float m_used = -INFINITY;
      float l = 0.f;
      bool ok = true;
      for (int kt = 0; kt < nkv_x; ++kt) {
        if (!warp_wait(&s_full[x], scnt & 1, ctl)) { ok = false; break; }
        ++scnt;
        tc_fence_after();
        // the whole score tile into registers, then S goes back to the issuer
        uint32_t sr[128];
        tmem_ld32p(t_s, &sr[0]);
        tmem_ld32p(t_s + 32, &sr[32]);
        tmem_ld32p(t_s + 64, &sr[64]);
        tmem_ld32p(t_s + 96, &sr[96]);
        tmem_ld_wait();
        reg_fence32(&sr[0]);
        reg_fence32(&sr[32]);
        reg_fence32(&sr[64]);
        reg_fence32(&sr[96]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(s_free);
        float* sv = reinterpret_cast<float*>(sr);
        const int kbase = kt * kAttnBN;
        if (kbase + kAttnBN - 1 > p0_x) {  // some key may lie past this row
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (kbase + i > qpos) sv[i] = -INFINITY;
        }
        // The row's first tile sets the offset m_used (its maximum); later
        // tiles reuse it without a maximum pass, which is exact (the final
        // division by the row sum cancels the common factor) while every
        // probability fits fp16.  The fp32 row sum bounds the largest
        // probability: past 2^15 the tile takes the rare path, which
        // recomputes the row's scores from Q and K in global memory and moves
        // the offset to their maximum.
        float f = 1.0f;
        bool need = false;
        if (kt == 0) m_used = attn_row_max(sv) * sl2;
        uint32_t P[64];
        float lt = attn_exp_pack(sv, sl2, m_used, P);
        if (kt > 0 && !(lt <= 32768.0f)) {
          float srow[128];  // local memory: the registers of sv stay registers
          int it_r = it;
          asm volatile("" : "+r"(it_r));  // decoded here, not kept live across the loop
          const AttnItem wr = attn_decode(p, it_r);
          attn_scores_from_global<HD>(p, wr.head, wr.t[x].m0 + row, kbase, qpos, row < wr.t[x].nvalid, srow);
          const float mt = fmaxf(attn_row_max(srow) * sl2, m_used);
          f = ex2_approx(m_used - mt);
          m_used = mt;
          need = true;
          lt = attn_exp_pack(srow, sl2, m_used, P);
        }
        // P_x and O_x are free once the previous PV of this tile has finished
        if (kt > 0) {
          if (!warp_wait(&pv_done[x], pvcnt & 1, ctl)) { ok = false; break; }
          ++pvcnt;
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
            // rare: rescale O to the new maximum before the next PV adds to it
#pragma unroll 1
            for (int j = 0; j < HD / 32; ++j) {
              uint32_t r[32];
              tmem_ld32(t_o + j * 32, r);
              tmem_ld_wait();
#pragma unroll
              for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * f);
              tmem_st32(t_o + j * 32, r);
            }
          }
        }
        // keys 2c, 2c+1 -> column c of P
        tmem_st32p(t_p, &P[0]);
        tmem_st32p(t_p + 32, &P[32]);
        l = l * f + lt;
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      int it_e = it;
      asm volatile("" : "+r"(it_e));
      const AttnItem w = attn_decode(p, it_e);
      const AttnTile T = w.t[x];
      const bool row_valid = row < T.nvalid;
      // epilogue: O / l -> fp16 -> A[m0 + row, head]
      if (!warp_wait(&o_full[x], icnt & 1, ctl)) break;
      ++icnt;
      tc_fence_after();
      const float inv = 1.0f / l;
      if (p.lse != nullptr && row_valid) {
        const int chunk = T.m0 >= p.c ? 1 : 0;
        const int li = (T.m0 - chunk * p.c) + row;
        if (dbg_ok(w.head < p.H && li < p.c, p.status))
          p.lse[(w.head * 2 + chunk) * p.c_pad + li] = m_used + lg2_approx(l);
      }
      __half* dst = p.out + static_cast<int64_t>(T.m0 + row) * p.ldo + w.head * HD;
#pragma unroll
      for (int j = 0; j < HD / 32; ++j) {
        uint32_t r[32];
        tmem_ld32(t_o + j * 32, r);
        tmem_ld_wait();
        if (row_valid && dbg_ok(T.m0 + row < 2 * p.c && (w.head + 1) * HD <= p.ldo, p.status)) {
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
      if (lane == 0) mbar_arrive(&o_free[x]);
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
