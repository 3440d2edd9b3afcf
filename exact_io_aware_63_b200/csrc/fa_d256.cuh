// fa_d256.cuh - head dimension 256.
//
// The same method as the 64- and 128-column kernels (tiles that fit on chip,
// an online softmax in the forward pass, recomputation of the score tiles in
// the backward pass: "FlashAttention: Fast and Memory-Efficient Exact
// Attention with IO-Awareness", opendecode.dev summary, "The key idea";
// "FlashAttention, Decoded", "The Hardware Picture"), laid out for tiles
// whose rows are 512 bytes: a 128 x 256 bf16 tile takes 64 KB of shared
// memory and a 128 x 256 float32 accumulator half of tensor memory.
//
// Shared memory holds one such tile per work unit (the unit's own query tile
// in the forward pass) and streams the other operands through one ring of
// 16 KB chunks, each consumed by the MMAs in the order the producer loaded it:
//  * a column chunk: rows r0 .. r0+127, columns 64c .. 64c+63 (one 64-column
//    TMA box, 128-byte swizzled rows): the K-major operand slice of a
//    contraction over the head dimension (4 MMA steps of 16 columns);
//  * a row chunk: rows r0+32m .. r0+32m+31, all 256 columns (four 64-column
//    boxes of 32 rows): the MN-major operand of a contraction over rows
//    (2 MMA steps of 16 rows, N = 256).
//
// Forward kernel (one persistent CTA per SM, 8 warps):
//   warp 0      TMA producer: Q_i (four boxes), then the chunks of each
//               visited key tile: K_j as column chunks, V_j as row chunks
//   warp 1      TMEM owner and MMA issuer (one thread)
//   warps 4-7   softmax warpgroup, one query row per thread (TMEM lane)
// A unit is one 128-row query tile.  TMEM: S double-buffered in columns
// [0,128) and [128,256) (P, bf16, written over the first 64 columns of its
// S), O in [256,512).  Issue order S(0) S(1) PV(0) S(2) PV(1) ...: the MMAs
// of S(k+1) run while the softmax of tile k runs.  Per key tile the tensor
// core does 2 x 128 x 128 x 256 MACs (S and P V, 2048 cycles at full rate)
// against about 1000 cycles of softmax for the warpgroup, so one softmax
// warpgroup keeps up.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

constexpr int k256Chunk = 16384;  // bytes of one ring chunk

struct Fwd256Cfg {
  static constexpr int D = 256;
  static constexpr int kThreads = 256;
  static constexpr int kTileBytes = kTile * D * 2;  // 64 KB
  static constexpr int kRing = 9;                   // chunks in flight
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = kOffQ + kTileBytes;
  static constexpr int kOffBar = kOffRing + kRing * k256Chunk;
  // q_full, q_empty, ring_full[R], ring_empty[R], s_full[2], p_full, pv_done, drain,
  // staged (the softmax warpgroup's output rows are in shared memory)
  static constexpr int kNumBars = 8 + 2 * kRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColO = 256;
  __device__ static constexpr uint32_t col_s(int b) { return b ? 128u : 0u; }
};

// Shared-memory descriptors of the two chunk kinds and of a resident tile:
// K-major 64-column boxes (8-row groups 1024 bytes apart), and MN-major row
// chunks whose four 64-column groups lie 4096 bytes apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t saddr) { return sw128_desc(saddr, 16, 1024); }
__device__ __forceinline__ uint64_t desc_rowchunk(uint32_t saddr) {
  return sw128_desc(saddr, 4096, 1024);
}

template <bool kUnused = false>
__global__ void __launch_bounds__(Fwd256Cfg::kThreads, 1)
    fa_fwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v32,
                     const __grid_constant__ CUtensorMap tm_o, const FwdParams p) {
  using Cfg = Fwd256Cfg;
  constexpr int R = Cfg::kRing;
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_launch_dependents();
  if (!smem_aligned_1024(smem)) return;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::kOffBar;
  const uint32_t q_full = bar0, q_empty = bar0 + 8;
  auto ring_full = [&](int s) { return bar0 + 8 * (2 + s); };
  auto ring_empty = [&](int s) { return bar0 + 8 * (2 + R + s); };
  auto s_full = [&](int b) { return bar0 + 8 * (2 + 2 * R + b); };
  const uint32_t p_full = bar0 + 8 * (4 + 2 * R);
  const uint32_t pv_done = bar0 + 8 * (5 + 2 * R);
  const uint32_t drain_bar = bar0 + 8 * (6 + 2 * R);
  const uint32_t staged = bar0 + 8 * (7 + 2 * R);
  static_assert(Cfg::kNumBars == 8 + 2 * R, "barrier layout");
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  auto chunk = [&](uint32_t c) { return sbase + Cfg::kOffRing + (c % R) * k256Chunk; };

  const int warp = warp_id();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(staged, 128);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(ring_full(s), 1);
      mbar_init(ring_empty(s), 1);
    }
    mbar_init(s_full(0), 1);
    mbar_init(s_full(1), 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v32);
    prefetch_tmap(&tm_o);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_base_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_base_slot;
  const int G = gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t units = 0, chunks = 0;
      bool ok = true;
      // one chunk: wait for its ring slot, then load it (1 box or 4 boxes)
      auto load_k = [&](const FwdUnit& w, int j, int c) -> bool {
        const uint32_t s = chunks % R;
        if (!mbar_wait(ring_empty(s), ((chunks / R) & 1) ^ 1)) return false;
        mbar_arrive_expect_tx(ring_full(s), k256Chunk);
        tma_load_3d(chunk(chunks), &tm_k, 64 * c, j * kTile, w.tz, ring_full(s));
        ++chunks;
        return true;
      };
      auto load_v = [&](const FwdUnit& w, int j, int m) -> bool {
        const uint32_t s = chunks % R;
        if (!mbar_wait(ring_empty(s), ((chunks / R) & 1) ^ 1)) return false;
        mbar_arrive_expect_tx(ring_full(s), k256Chunk);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(chunk(chunks) + 4096 * c, &tm_v32, 64 * c, j * kTile + 32 * m, w.tz,
                      ring_full(s));
        ++chunks;
        return true;
      };
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode<false>(p, u);
        ok = mbar_wait(q_empty, (units & 1) ^ 1);
        if (!ok) break;
        ++units;
        mbar_arrive_expect_tx(q_full, Cfg::kTileBytes);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(sbase + Cfg::kOffQ + 16384 * c, &tm_q, 64 * c, w.i0 * kTile, w.tz, q_full);
        // consumption order: K(v0) K(v1) V(v0) K(v2) V(v1) ... V(v_last)
        int jk = fwd_next(p, w, 0);  // visit k
        int jprev = -1;              // visit k - 1
        while (ok && (jk < w.j_end || jprev >= 0)) {
          if (jk < w.j_end)
            for (int c = 0; c < 4 && ok; ++c) ok = load_k(w, jk, c);
          if (jprev >= 0)
            for (int m = 0; m < 4 && ok; ++m) ok = load_v(w, jprev, m);
          jprev = (jk < w.j_end) ? jk : -1;
          if (jk < w.j_end) jk = fwd_next(p, w, jk + 1);
          if (*abort_flag) ok = false;
        }
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, 0, 1);
      uint32_t units = 0, chunks = 0, pcnt = 0;
      uint32_t scnt[2] = {0, 0};
      bool ok = true;
      auto wait_chunk = [&]() -> bool {
        return mbar_wait(ring_full(chunks % R), (chunks / R) & 1);
      };
      // S(k) = Q K_j^T into buffer b: four column chunks of K_j
      auto issue_s = [&](int b, const FwdUnit& w, int j) -> bool {
        for (int c = 0; c < 4; ++c) {
          if (!wait_chunk()) return false;
          tc_fence_after();
          const uint64_t dq = desc_kmajor(sbase + Cfg::kOffQ + 16384 * c);
          const uint64_t dk = desc_kmajor(chunk(chunks));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tmem + Cfg::col_s(b), dq + ((kk * 32) >> 4), dk + ((kk * 32) >> 4), idesc_s,
                    (c > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ring_empty(chunks % R));
          ++chunks;
        }
        umma_commit(s_full(b));
        ++scnt[b];
        if (p.visited) p.visited[((size_t)w.bh * p.n_t + w.i0) * p.n_t + j] = 1;
        return true;
      };
      // O (+)= P V_j from buffer b's P: four row chunks of V_j (32 keys each)
      auto issue_pv = [&](int b, bool first) -> bool {
        if (!mbar_wait(p_full, pcnt & 1)) return false;
        ++pcnt;
        for (int m = 0; m < 4; ++m) {
          if (!wait_chunk()) return false;
          tc_fence_after();
          const uint64_t dv = desc_rowchunk(chunk(chunks));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts(tmem + Cfg::kColO, tmem + Cfg::col_s(b) + (2 * m + kk) * 8,
                    dv + ((kk * 2048) >> 4), idesc_pv, (!first || m > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ring_empty(chunks % R));
          ++chunks;
        }
        umma_commit(pv_done);
        return true;
      };
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode<false>(p, u);
        ok = mbar_wait(q_full, units & 1);
        ++units;
        if (!ok) break;
        int jk = fwd_next(p, w, 0);
        int k = 0;
        bool have_prev = false;
        while (ok && (jk < w.j_end || have_prev)) {
          if (jk < w.j_end) ok = issue_s(k & 1, w, jk);
          if (ok && have_prev) ok = issue_pv((k - 1) & 1, k == 1);
          have_prev = jk < w.j_end;
          if (jk < w.j_end) jk = fwd_next(p, w, jk + 1);
          ++k;
          if (*abort_flag) ok = false;
        }
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tO = t_lane + Cfg::kColO;
    uint32_t units = 0, pv_cnt = 0;
    uint32_t scnt[2] = {0, 0};
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int u = unit_for_round(round, blockIdx.x, G);
      if (u >= p.num_units) break;
      const FwdUnit w = fwd_decode<false>(p, u);
      const uint32_t q_par = units & 1;
      ++units;
      const int row = w.i0 * kTile + r_local;
      float m_used = -INFINITY, l = 0.f;
      int k = 0;
      for (int j = fwd_next(p, w, 0); j < w.j_end; j = fwd_next(p, w, j + 1), ++k) {
        const int b = k & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(b), scnt[b] & 1));
        ++scnt[b];
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = t_lane + Cfg::col_s(b);
        float sv[kTile];
        {
          uint32_t r[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, r[c]);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            reg_fence32(r[c]);
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[c * 32 + e] = __uint_as_float(r[c][e]);
          }
        }
        // element masks on boundary tiles only (causal diagonal, keys past kv_len or N)
        const bool diag = p.causal && (j == w.i0);
        const int kv_lim = w.L - j * kTile;
        if (diag || kv_lim < kTile) {
          const int lim = diag ? min(r_local + 1, kv_lim) : kv_lim;
#pragma unroll
          for (int e = 0; e < kTile; ++e)
            if (e >= lim) sv[e] = -INFINITY;
        }
        float mx8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mx8[t] = fmaxf(sv[t], sv[t + 8]);
#pragma unroll
        for (int c = 16; c < kTile; c += 16)
#pragma unroll
          for (int t = 0; t < 8; ++t) mx8[t] = fmax3(mx8[t], sv[c + t], sv[c + 8 + t]);
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
        const float m_new = mx * p.scale_log2;
        float alpha = 1.f;
        bool rescale = false;
        if (k == 0) {
          m_used = m_new;
        } else if (m_new > m_used + kRescaleLog2) {
          alpha = ex2_approx(m_used - m_new);
          m_used = m_new;
          l *= alpha;
          rescale = true;
        }
        const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
        uint64_t ls4[4] = {0, 0, 0, 0};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t xx =
                f2_fma(f2_pack(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]), scale2, negm2);
            float x0, x1;
            f2_unpack(xx, x0, x1);
            const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            ls4[e & 3] = f2_add(ls4[e & 3], f2_pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        {
          const uint64_t s2 = f2_add(f2_add(ls4[0], ls4[1]), f2_add(ls4[2], ls4[3]));
          float s_lo, s_hi;
          f2_unpack(s2, s_lo, s_hi);
          l += s_lo + s_hi;
        }
        // the previous tile's P V must be complete before O may be rescaled
        if (k > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(pv_done, pv_cnt & 1));
          ++pv_cnt;
          if (!ok) break;
          tc_fence_after();
        }
        if (__any_sync(0xffffffffu, rescale)) {
          uint32_t r[32];
#pragma unroll 1
          for (int c = 0; c < 256 / 32; ++c) {
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      const int n_vis = k;
      if (n_vis > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(pv_done, pv_cnt & 1));
        ++pv_cnt;
        if (!ok) break;
        tc_fence_after();
      } else {
        // no key tile: the zeros below are staged over Q only after its load landed
        ok = __all_sync(0xffffffffu, mbar_wait(q_full, q_par));
        if (!ok) break;
      }
      const float inv_l = (n_vis > 0 && l > 0.f) ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 256 / 32; ++c) {
        uint32_t pk[16];
        if (n_vis > 0) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          reg_fence32(r);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l, __uint_as_float(r[2 * e + 1]) * inv_l);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = 0u;
        }
        // 64-column box c / 2, 16-byte granules 4 (c % 2) .. +3 of the row
        uint8_t* rowp = smem + Cfg::kOffQ + (c >> 1) * 16384 + r_local * 128;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int g = (c & 1) * 4 + v4;
          *reinterpret_cast<uint4*>(rowp + ((g ^ (r_local & 7)) << 4)) =
              make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
      }
      if (n_vis > 0) tc_fence_before();
      if (row < p.N)
        p.lse[(size_t)w.bh * p.N + row] = (n_vis > 0 && l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      // every row staged (a bounded wait: a warpgroup member that gave up earlier
      // never arrives, and the store is then skipped)
      fence_proxy_async_smem();
      mbar_arrive(staged);
      if (r_local == 0) {
        if (mbar_wait(staged, q_par)) {
          for (int c = 0; c < 4; ++c)
            tma_store_3d(&tm_o, 64 * c, w.i0 * kTile, w.tz, sbase + Cfg::kOffQ + 16384 * c);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(q_empty);  // Q's shared memory may be loaded again
        } else {
          *abort_flag = 1;
        }
      }
    }
    if (!ok) *abort_flag = 1;
    if (r_local == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

// ---------------------------------------------------------------------------
// Backward pass at head dimension 256: three persistent kernels after the
// preprocess kernel (D and the base-2 LSE, as for the other head sizes).
// dK and dV of a 128-key tile would need all 512 tensor-memory columns as
// float32 accumulators, leaving none for the score tiles, so each gradient
// has its own pass, each recomputing the score tile it needs on chip:
//   dQ pass (unit = query tile i, over its visited key tiles j in order):
//       S = Q_i K_j^T, dP = dO_i V_j^T, P = exp2(S s log2e - LSE2),
//       dS = P o (dP - D),  dQ_i += dS K_j          -> dQ = bf16(scale dQ_i)
//   dK pass (unit = key tile j, over its visited query tiles i):
//       S^T = K_j Q_i^T, dP^T = V_j dO_i^T, dS^T as above,
//       dK_j += dS^T Q_i                            -> dK = bf16(scale dK_j)
//   dV pass (unit = key tile j):
//       S^T = K_j Q_i^T (double-buffered), P^T,  dV_j += P^T dO_i -> bf16
// That is 8 products of 128 x 128 x 256 per (query tile, key tile) pair where
// one pass with room for everything would do 5; dQ has no atomics and every
// sum is taken in a fixed order, so the result is bitwise reproducible.
// Each pass keeps its unit's own tiles resident (Q_i and dO_i, or K_j and
// V_j) and streams the others through the 16 KB chunk ring.  TMEM: the score
// tile in [0,128), dP in [128,256) (dV pass: a second score buffer), the
// accumulator in [256,512); the bf16 P or dS operand of the accumulating MMA
// is written over the first 64 columns of its score tile.
// ---------------------------------------------------------------------------
enum Bwd256Mode : int { kPassDQ = 0, kPassDK = 1, kPassDV = 2 };

struct Bwd256Params {
  FwdParams q;        // dQ pass: query-tile units (masks, shape, unit order)
  BwdParams k;        // dK / dV passes: key-tile units; delta, lse2, dk, dv
  uint16_t* dq;
};

struct Bwd256Cfg {
  static constexpr int D = 256;
  // warps 0-3: producer, MMA issuer (TMEM owner), two idle; warps 4-11: two math
  // warpgroups, warpgroup h on score columns 64h .. 64h + 63 of every row and on
  // output columns 128h .. 128h + 127 in the epilogue
  static constexpr int kThreads = 384;
  static constexpr int kMathThreads = 256;
  static constexpr int kTileBytes = kTile * D * 2;  // 64 KB
  static constexpr int kOffA = 0;                   // resident tile A: Q_i or K_j
  static constexpr int kOffB = kTileBytes;          // resident tile B: dO_i or V_j
  static constexpr int kRing = 6;
  static constexpr int kOffRing = 2 * kTileBytes;
  static constexpr int kRowBytes = kTile * 4;
  static constexpr int kOffRow = kOffRing + kRing * k256Chunk;  // 2 slots x (-LSE2, -D)
  static constexpr int kOffBar = kOffRow + 2 * 2 * kRowBytes;
  // a_full, a_empty, ring_full[R], ring_empty[R], row_full[2], row_empty[2],
  // s_full[2], p_full, acc_done, drain, staged, dp_free
  static constexpr int kNumBars = 13 + 2 * kRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;
};

template <int kMode>
__global__ void __launch_bounds__(Bwd256Cfg::kThreads, 1)
    fa_bwd256_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_q32,
                     const __grid_constant__ CUtensorMap tm_k32,
                     const __grid_constant__ CUtensorMap tm_do32,
                     const __grid_constant__ CUtensorMap tm_out, const Bwd256Params bp) {
  using Cfg = Bwd256Cfg;
  constexpr int R = Cfg::kRing;
  constexpr bool kRowUnits = (kMode == kPassDQ);  // units are query tiles
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_launch_dependents();
  if (!smem_aligned_1024(smem)) return;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::kOffBar;
  const uint32_t a_full = bar0, a_empty = bar0 + 8;
  auto ring_full = [&](int s) { return bar0 + 8 * (2 + s); };
  auto ring_empty = [&](int s) { return bar0 + 8 * (2 + R + s); };
  auto row_full = [&](int s) { return bar0 + 8 * (2 + 2 * R + s); };
  auto row_empty = [&](int s) { return bar0 + 8 * (4 + 2 * R + s); };
  auto s_full = [&](int b) { return bar0 + 8 * (6 + 2 * R + b); };
  const uint32_t p_full = bar0 + 8 * (8 + 2 * R);    // P / dS written by the math warps
  const uint32_t acc_done = bar0 + 8 * (9 + 2 * R);  // the unit's accumulator complete
  const uint32_t drain_bar = bar0 + 8 * (10 + 2 * R);
  const uint32_t staged = bar0 + 8 * (11 + 2 * R);  // the unit's output rows are staged
  // dQ / dK passes: the math warps hold the tile's dP in registers
  const uint32_t dp_free = bar0 + 8 * (12 + 2 * R);
  static_assert(Cfg::kNumBars == 13 + 2 * R, "barrier layout");
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  auto chunk = [&](uint32_t c) { return sbase + Cfg::kOffRing + (c % R) * k256Chunk; };
  const FwdParams& pq = bp.q;
  const BwdParams& pk = bp.k;

  const int warp = warp_id();
  const int lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(a_full, 1);
    mbar_init(a_empty, 1);
    for (int s = 0; s < R; ++s) {
      mbar_init(ring_full(s), 1);
      mbar_init(ring_empty(s), 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(row_full(s), 1);
      mbar_init(row_empty(s), 8);  // lane 0 of each math warp
      mbar_init(s_full(s), 1);
    }
    mbar_init(p_full, Cfg::kMathThreads);
    mbar_init(acc_done, 1);
    mbar_init(drain_bar, 1);
    mbar_init(staged, Cfg::kMathThreads);
    mbar_init(dp_free, Cfg::kMathThreads);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_out);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_base_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait();
  const uint32_t tmem = *tmem_base_slot;
  const int G = gridDim.x;
  const int num_units = kRowUnits ? pq.num_units : pk.num_units;

  // Unit u and its visits, for every role alike.  Query-tile units: the
  // visited key tiles of query tile i0 (fwd_next); key-tile units: the
  // visited query tiles of key tile j (bwd_next).
  struct Unit {
    FwdUnit f;
    BwdUnit b;
  };
  auto decode = [&](int u) {
    Unit w;
    if constexpr (kRowUnits) w.f = fwd_decode<false>(pq, u);
    else w.b = bwd_decode<false>(pk, u);
    return w;
  };
  auto first_visit = [&](const Unit& w) {
    if constexpr (kRowUnits) return fwd_next(pq, w.f, 0);
    else return w.b.i_first;
  };
  auto next_visit = [&](const Unit& w, int t) {
    if constexpr (kRowUnits) return fwd_next(pq, w.f, t + 1);
    else return bwd_next(pk, w.b, t + 1);
  };
  auto end_visit = [&](const Unit& w) {
    if constexpr (kRowUnits) return w.f.j_end;
    else return w.b.n_tq;
  };
  auto head = [&](const Unit& w) {
    if constexpr (kRowUnits) return w.f.bh;
    else return w.b.bh;
  };
  auto own_tile = [&](const Unit& w) {
    if constexpr (kRowUnits) return w.f.i0;
    else return w.b.j;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t units = 0, chunks = 0, rows = 0;
      bool ok = true;
      auto slot = [&]() -> bool {
        return mbar_wait(ring_empty(chunks % R), ((chunks / R) & 1) ^ 1);
      };
      // column chunk c (64 columns, 128 rows from row0) of a tensor
      auto load_col = [&](const CUtensorMap* tm, int row0, int z, int c) -> bool {
        if (!slot()) return false;
        const int s = chunks % R;
        mbar_arrive_expect_tx(ring_full(s), k256Chunk);
        tma_load_3d(chunk(chunks), tm, 64 * c, row0, z, ring_full(s));
        ++chunks;
        return true;
      };
      // row chunk m (32 rows from row0 + 32 m, all 256 columns) of a tensor
      auto load_row = [&](const CUtensorMap* tm32, int row0, int z, int m) -> bool {
        if (!slot()) return false;
        const int s = chunks % R;
        mbar_arrive_expect_tx(ring_full(s), k256Chunk);
        for (int c = 0; c < 4; ++c)
          tma_load_3d(chunk(chunks) + 4096 * c, tm32, 64 * c, row0 + 32 * m, z, ring_full(s));
        ++chunks;
        return true;
      };
      // the query tile's -LSE2 and -D rows (key-tile units)
      auto load_rows = [&](int bh, int i) -> bool {
        const int s = rows & 1;
        if (!mbar_wait(row_empty(s), ((rows >> 1) & 1) ^ 1)) return false;
        const long long qrow = (long long)bh * pk.n_t * kTile + (long long)i * kTile;
        mbar_arrive_expect_tx(row_full(s), 2 * Cfg::kRowBytes);
        bulk_load(sbase + Cfg::kOffRow + s * 2 * Cfg::kRowBytes, pk.lse2 + qrow, Cfg::kRowBytes,
                  row_full(s));
        bulk_load(sbase + Cfg::kOffRow + s * 2 * Cfg::kRowBytes + Cfg::kRowBytes, pk.delta + qrow,
                  Cfg::kRowBytes, row_full(s));
        ++rows;
        return true;
      };
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= num_units) break;
        const Unit w = decode(u);
        const int z = head(w);
        const int r0 = own_tile(w) * kTile;
        ok = mbar_wait(a_empty, (units & 1) ^ 1);
        if (!ok) break;
        ++units;
        // resident tiles: Q_i and dO_i (dQ pass), K_j and V_j (dK), K_j (dV)
        const int nres = (kMode == kPassDV) ? 1 : 2;
        mbar_arrive_expect_tx(a_full, nres * Cfg::kTileBytes);
        for (int c = 0; c < 4; ++c) {
          tma_load_3d(sbase + Cfg::kOffA + 16384 * c, kRowUnits ? &tm_q : &tm_k, 64 * c, r0, z,
                      a_full);
          if (nres == 2)
            tma_load_3d(sbase + Cfg::kOffB + 16384 * c, kRowUnits ? &tm_do : &tm_v, 64 * c, r0, z,
                        a_full);
        }
        if constexpr (kMode == kPassDV) {
          // consumption order: Q^(v0) Q^(v1) dO(v0) Q^(v2) dO(v1) ... dO(v_last)
          int t = first_visit(w), tprev = -1;
          while (ok && (t < end_visit(w) || tprev >= 0)) {
            if (t < end_visit(w)) {
              ok = load_rows(z, t);
              for (int c = 0; c < 4 && ok; ++c) ok = load_col(&tm_q, t * kTile, z, c);
            }
            if (tprev >= 0)
              for (int m = 0; m < 4 && ok; ++m) ok = load_row(&tm_do32, tprev * kTile, z, m);
            tprev = (t < end_visit(w)) ? t : -1;
            if (t < end_visit(w)) t = next_visit(w, t);
            if (*abort_flag) ok = false;
          }
        } else {
          // S: K_j (dQ pass) or Q_i (dK pass) columns; dP: V_j or dO_i columns;
          // the accumulating product: K_j or Q_i rows.  Consumption order
          // (dP one visit ahead): S(v0) dP(v0) | dP(v1) rows(v0) S(v1) | ...
          const CUtensorMap* tm_s = (kMode == kPassDQ) ? &tm_k : &tm_q;
          const CUtensorMap* tm_dp = (kMode == kPassDQ) ? &tm_v : &tm_do;
          const CUtensorMap* tm_acc = (kMode == kPassDQ) ? &tm_k32 : &tm_q32;
          int t = first_visit(w);
          if (t < end_visit(w)) {
            if constexpr (kMode == kPassDK) ok = load_rows(z, t);
            for (int c = 0; c < 4 && ok; ++c) ok = load_col(tm_s, t * kTile, z, c);
            for (int c = 0; c < 4 && ok; ++c) ok = load_col(tm_dp, t * kTile, z, c);
          }
          while (ok && t < end_visit(w)) {
            const int tn = next_visit(w, t);
            const bool more = tn < end_visit(w);
            if (more)
              for (int c = 0; c < 4 && ok; ++c) ok = load_col(tm_dp, tn * kTile, z, c);
            for (int m = 0; m < 4 && ok; ++m) ok = load_row(tm_acc, t * kTile, z, m);
            if (more && ok) {
              if constexpr (kMode == kPassDK) ok = load_rows(z, tn);
              for (int c = 0; c < 4 && ok; ++c) ok = load_col(tm_s, tn * kTile, z, c);
            }
            t = tn;
            if (*abort_flag) ok = false;
          }
        }
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, 256, 0, 1);
      uint32_t units = 0, chunks = 0, pcnt = 0, dpcnt = 0;
      bool ok = true;
      auto wait_chunk = [&]() -> bool {
        return mbar_wait(ring_full(chunks % R), (chunks / R) & 1);
      };
      // D[col] (+)= resident tile (A or B area) x streamed column chunks, over 256
      auto issue_cols = [&](uint32_t col, int area, bool acc) -> bool {
        for (int c = 0; c < 4; ++c) {
          if (!wait_chunk()) return false;
          tc_fence_after();
          const uint64_t da = desc_kmajor(sbase + area + 16384 * c);
          const uint64_t db = desc_kmajor(chunk(chunks));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_ss(tmem + col, da + ((kk * 32) >> 4), db + ((kk * 32) >> 4), idesc_s,
                    (acc || c > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ring_empty(chunks % R));
          ++chunks;
        }
        return true;
      };
      // accumulator (+)= (bf16 operand in TMEM at col_a) x streamed row chunks (N = 256)
      auto issue_rows = [&](uint32_t col_a, bool first) -> bool {
        for (int m = 0; m < 4; ++m) {
          if (!wait_chunk()) return false;
          tc_fence_after();
          const uint64_t db = desc_rowchunk(chunk(chunks));
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            umma_ts(tmem + Cfg::kColAcc, tmem + col_a + (2 * m + kk) * 8, db + ((kk * 2048) >> 4),
                    idesc_acc, (!first || m > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ring_empty(chunks % R));
          ++chunks;
        }
        return true;
      };
      uint32_t scnt[2] = {0, 0};
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= num_units) break;
        const Unit w = decode(u);
        ok = mbar_wait(a_full, units & 1);
        ++units;
        if (!ok) break;
        tc_fence_after();
        int n = 0;  // visits issued
        if constexpr (kMode == kPassDV) {
          int t = first_visit(w);
          bool have_prev = false;
          int k = 0;
          while (ok && (t < end_visit(w) || have_prev)) {
            if (t < end_visit(w)) {
              const int b = k & 1;
              ok = issue_cols(b ? 128u : 0u, Cfg::kOffA, false);
              if (!ok) break;
              umma_commit(s_full(b));
              ++scnt[b];
              if (pk.visited) pk.visited[((size_t)w.b.bh * pk.n_t + t) * pk.n_t + w.b.j] = 1;
            }
            if (have_prev) {
              ok = mbar_wait(p_full, pcnt & 1);
              ++pcnt;
              if (!ok) break;
              tc_fence_after();
              ok = issue_rows(((k - 1) & 1) ? 128u : 0u, k == 1);
            }
            have_prev = t < end_visit(w);
            if (t < end_visit(w)) t = next_visit(w, t);
            ++k;
            if (*abort_flag) ok = false;
          }
          n = k > 0 ? k - 1 : 0;  // the unit's visits: the last step issued only dV
        } else {
          auto mark = [&](int t) {
            if constexpr (kRowUnits) {
              if (pq.visited) pq.visited[((size_t)w.f.bh * pq.n_t + w.f.i0) * pq.n_t + t] = 1;
            } else {
              if (pk.visited) pk.visited[((size_t)w.b.bh * pk.n_t + t) * pk.n_t + w.b.j] = 1;
            }
          };
          // Per visit: dP of the next visit as soon as the math warps hold this
          // one's dP in registers (its MMAs overlap their dS work), then the
          // accumulating product once dS is in TMEM, then the next score tile
          // over that dS (issue order).
          int t = first_visit(w);
          if (t < end_visit(w)) {
            ok = issue_cols(Cfg::kColS, Cfg::kOffA, false) &&
                 issue_cols(Cfg::kColDP, Cfg::kOffB, false);
            if (ok) {
              umma_commit(s_full(0));
              mark(t);
            }
          }
          while (ok && t < end_visit(w)) {
            const int tn = next_visit(w, t);
            const bool more = tn < end_visit(w);
            ok = mbar_wait(dp_free, dpcnt & 1);
            ++dpcnt;
            if (!ok) break;
            tc_fence_after();
            if (more) {
              ok = issue_cols(Cfg::kColDP, Cfg::kOffB, false);
              if (!ok) break;
            }
            // dS (bf16, over the score tile) x streamed rows into the accumulator
            ok = mbar_wait(p_full, pcnt & 1);
            ++pcnt;
            if (!ok) break;
            tc_fence_after();
            ok = issue_rows(Cfg::kColS, n == 0);
            ++n;
            if (!ok) break;
            if (more) {
              ok = issue_cols(Cfg::kColS, Cfg::kOffA, false);
              if (!ok) break;
              umma_commit(s_full(0));
              mark(tn);
            }
            t = tn;
            if (*abort_flag) ok = false;
          }
        }
        if (!ok) break;
        if (n > 0) umma_commit(acc_done);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ math warpgroups
    const int hg = (warp - 4) >> 2;  // warpgroup: score chunks 2hg, 2hg + 1
    const int quarter = warp & 3;
    const int rl = quarter * 32 + lane;  // row within the unit's tile = TMEM lane
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    uint32_t units = 0, rows = 0, acc_cnt = 0;
    uint32_t scnt[2] = {0, 0};
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int u = unit_for_round(round, blockIdx.x, G);
      if (u >= num_units) break;
      const Unit w = decode(u);
      const uint32_t a_par = units & 1;
      ++units;
      const int bh = head(w);
      const int me = own_tile(w) * kTile + rl;  // this thread's row (query or key index)
      // dQ pass: this query row's -LSE2 and -D (per-head padded layout)
      float my_nlse2 = 0.f, my_nd = 0.f;
      int kv_L = 0;  // dQ pass: keys c >= kv_L are padding
      if constexpr (kRowUnits) {
        const long long prow = (long long)bh * pq.n_t * kTile + me;
        my_nlse2 = __ldg(pk.lse2 + prow);
        my_nd = __ldg(pk.delta + prow);
        kv_L = w.f.L;
      }
      const bool key_valid = kRowUnits ? true : (me < w.b.L);
      int n = 0, k = 0;
      for (int t = first_visit(w); t < end_visit(w); t = next_visit(w, t), ++k) {
        const int b = (kMode == kPassDV) ? (k & 1) : 0;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(b), scnt[b] & 1));
        ++scnt[b];
        if (!ok) break;
        const float4* nl4 = nullptr;
        const float4* nd4 = nullptr;
        int rs = 0;
        if constexpr (!kRowUnits) {
          rs = rows & 1;
          ok = __all_sync(0xffffffffu, mbar_wait(row_full(rs), (rows >> 1) & 1));
          ++rows;
          if (!ok) break;
          nl4 = reinterpret_cast<const float4*>(smem + Cfg::kOffRow + rs * 2 * Cfg::kRowBytes);
          nd4 = reinterpret_cast<const float4*>(smem + Cfg::kOffRow + rs * 2 * Cfg::kRowBytes +
                                                Cfg::kRowBytes);
        }
        tc_fence_after();
        const uint32_t tS = t_lane + (b ? 128u : 0u);
        const uint32_t tDP = t_lane + Cfg::kColDP;
        // element mask of this tile: allowed(query, key) for this thread's row
        //   dQ pass: row = query me, columns = keys t*128 + e
        //   dK / dV: row = key me, columns = queries t*128 + e
        const int col0 = t * kTile;
        // tiles with no element mask for this warp's rows take a path without the
        // per-element tests
        const bool row_interior =
            kRowUnits ? (col0 + kTile <= kv_L && (!pq.causal || col0 + kTile - 1 <= me))
                      : (key_valid && (!pk.causal || me <= col0));
        const bool interior = __all_sync(0xffffffffu, row_interior);
        // chunk c (32 columns): S (and dP) from TMEM, bf16 P or dS back over the
        // score tile's first columns.  The loads of chunk c + 1 are issued before
        // chunk c is computed, so their latency overlaps it.
        // dQ / dK passes: all of dP into registers first; the issuer then
        // computes the next visit's dP while this tile's dS is formed
        // this warpgroup's two chunks of 32 columns: c0 and c0 + 1
        const int c0 = 2 * hg;
        uint32_t rs_[2][32], rd[kMode != kPassDV ? 2 : 1][32];
        if constexpr (kMode != kPassDV) {
#pragma unroll
          for (int i = 0; i < 2; ++i) tmem_ld32(tDP + 32 * (c0 + i), rd[i]);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 2; ++i) reg_fence32(rd[i]);
          tc_fence_before();
          mbar_arrive(dp_free);
        }
        auto load = [&](int i) { tmem_ld32(tS + 32 * (c0 + i), rs_[i]); };
        auto compute = [&](int i, auto interior_tag) {
          const int c = c0 + i;
          constexpr bool kInterior = decltype(interior_tag)::value;
          uint32_t pk16[16];
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            float4 nl4v, nd4v;
            if constexpr (kRowUnits) {
              nl4v = make_float4(my_nlse2, my_nlse2, my_nlse2, my_nlse2);
              nd4v = make_float4(my_nd, my_nd, my_nd, my_nd);
            } else {
              nl4v = nl4[8 * c + e4];
              nd4v = nd4[8 * c + e4];
            }
            const float nlv[4] = {nl4v.x, nl4v.y, nl4v.z, nl4v.w};
            [[maybe_unused]] const float ndv[4] = {nd4v.x, nd4v.y, nd4v.z, nd4v.w};
            float v[4];
#pragma unroll
            for (int h = 0; h < 4; ++h) {
              const int e = 4 * e4 + h;
              float pv = ex2_approx(fmaf(__uint_as_float(rs_[i][e]), pk.scale_log2, nlv[h]));
              if constexpr (!kInterior) {
                const int col = col0 + 32 * c + e;  // key (dQ pass) or query index
                const bool allowed = kRowUnits ? (col < kv_L && (!pq.causal || col <= me))
                                               : (key_valid && (!pk.causal || me <= col));
                pv = allowed ? pv : 0.f;
              }
              if constexpr (kMode == kPassDV) {
                v[h] = pv;
              } else {
                // dS = P (dP - D), with P rounded to bf16 as the other kernels use it
                const float pr = __bfloat162float(__float2bfloat16_rn(pv));
                v[h] = pr * (__uint_as_float(rd[kMode != kPassDV ? i : 0][e]) + ndv[h]);
              }
            }
            pk16[2 * e4] = pack_bf16x2(v[0], v[1]);
            pk16[2 * e4 + 1] = pack_bf16x2(v[2], v[3]);
          }
          tmem_st16(tS + 16 * c, pk16);
        };
        load(0);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          tmem_wait_ld();
          reg_fence32(rs_[i]);
          if (i == 0) load(1);
          if (interior)
            compute(i, std::true_type{});
          else
            compute(i, std::false_type{});
        }
        if constexpr (!kRowUnits) {
          __syncwarp();
          if (lane == 0) mbar_arrive(row_empty(rs));
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        ++n;
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) break;
      // ---------------------------------------------------------------- epilogue
      if (n > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(acc_done, acc_cnt & 1));
        ++acc_cnt;
      } else {
        ok = __all_sync(0xffffffffu, mbar_wait(a_full, a_par));
      }
      if (!ok) break;
      tc_fence_after();
      const float mul = (kMode == kPassDV) ? 1.f : pk.scale;
#pragma unroll 1
      for (int c = 4 * hg; c < 4 * hg + 4; ++c) {
        uint32_t pk16[16];
        if (n > 0) {  // warp-uniform: tcgen05.ld is a collective of the whole warp
          uint32_t r[32];
          tmem_ld32(t_lane + Cfg::kColAcc + 32 * c, r);
          tmem_wait_ld();
          reg_fence32(r);
          // key rows past kv_len or N get zeros (their accumulator rows are zero
          // already: every P^T entry of such a row is masked)
          const float m2 = key_valid ? mul : 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk16[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * m2, __uint_as_float(r[2 * e + 1]) * m2);
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) pk16[e] = 0u;
        }
        uint8_t* rowp = smem + Cfg::kOffA + (c >> 1) * 16384 + rl * 128;
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const int g = (c & 1) * 4 + v4;
          *reinterpret_cast<uint4*>(rowp + ((g ^ (rl & 7)) << 4)) =
              make_uint4(pk16[4 * v4], pk16[4 * v4 + 1], pk16[4 * v4 + 2], pk16[4 * v4 + 3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      mbar_arrive(staged);
      if (hg == 0 && rl == 0) {
        if (mbar_wait(staged, a_par)) {
          for (int c = 0; c < 4; ++c)
            tma_store_3d(&tm_out, 64 * c, own_tile(w) * kTile, bh, sbase + Cfg::kOffA + 16384 * c);
          bulk_commit_group();
          bulk_wait_group_read0();
          mbar_arrive(a_empty);  // the resident tiles may be loaded again
        } else {
          *abort_flag = 1;
        }
      }
    }
    if (!ok) *abort_flag = 1;
    if (hg == 0 && rl == 0) bulk_wait_group0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace fa
