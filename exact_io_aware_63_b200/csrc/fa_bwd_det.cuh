// fa_bwd_det.cuh - dQ without atomics, for a bitwise-reproducible backward.
//
// fa_bwd adds each key tile's dQ partial into a float32 accumulator with
// TMA reduce-adds, whose order across CTAs varies from run to run, so the
// rounding of dQ does too.  This kernel instead owns one query tile per work
// unit and walks that tile's visited key tiles in increasing order,
// recomputing what it needs on chip (the backward pass recomputes rather than
// stores: "FlashAttention, Decoded", "The Hardware Picture"):
//   S  = Q_i K_j^T,  dP = dO_i V_j^T               (tcgen05, float32 in TMEM)
//   P  = 2^(S * scale * log2 e - LSE2),  dS = P o (dP - D)
//   dQ_i += dS K_j                                  (accumulated in TMEM)
// and writes dQ_i = bf16(scale * dQ_i) once.  Every sum is taken in the same
// order on every run, so dQ is bitwise reproducible; dK and dV from the main
// kernel already are (one CTA owns each key tile).
//
// Roles (12 warps):
//   warp 0      TMA producer: Q_i, dO_i and the tile's -LSE2 / -D rows
//               (double-buffered across units for D = 64), then K_j, V_j of
//               each visited key tile through a kStages ring
//   warp 1      MMA issuer (one thread), TMEM owner
//   warps 4-11  two math warpgroups, one query row per thread (TMEM lane):
//               warpgroup h on keys 64h .. 64h + 63 of every key tile and on
//               dQ columns h D/2 .. (h + 1) D/2 - 1 in the epilogue
// TMEM columns: S [0,128), dP [128,256), dQ [256,256+D), dS (bf16, two per
// column) [384,448).
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct DetParams {
  FwdParams sched;     // masks, shape, unit order (the forward's one-tile units)
  const float* delta;  // -D per row
  const float* lse2;   // -LSE * log2(e) per row (-inf: row with no key)
  uint16_t* dq;
  float scale;
};

template <int D>
struct DetCfg {
  static constexpr int kThreads = 384;
  static constexpr int kMathThreads = 256;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kBoxes = D / 64;
  static constexpr int kQSlots = (D == 64) ? 2 : 1;  // Q_i + dO_i per slot
  static constexpr int kStages = (D == 64) ? 4 : 2;  // K_j + V_j per stage
  static constexpr int kRowBytes = kTile * 4;
  static constexpr int kOffQ = 0;                     // slot s: Q at +0, dO at +kTileBytes
  static constexpr int kOffK = kOffQ + kQSlots * 2 * kTileBytes;  // stage s: K, then V
  static constexpr int kOffRow = kOffK + kStages * 2 * kTileBytes;  // slot s: -LSE2, -D
  static constexpr int kOffBar = kOffRow + kQSlots * 2 * kRowBytes;
  // q_full[QS], q_empty[QS], k_full[S], k_empty[S], v_full[S], v_empty[S],
  // s_full, s_free, ds_full, ds_free, dq_full, drain
  static constexpr int kNumBars = 2 * kQSlots + 4 * kStages + 6;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 256, kColDS = 384;
};

template <int D>
__global__ void __launch_bounds__(DetCfg<D>::kThreads, 1)
    fa_bwd_dq_det_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_do, const DetParams dp) {
  using Cfg = DetCfg<D>;
  constexpr int S = Cfg::kStages;
  constexpr int QS = Cfg::kQSlots;
  const FwdParams& p = dp.sched;
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_launch_dependents();
  if (!smem_aligned_1024(smem)) return;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::kOffBar;
  auto q_full = [&](int s) { return bar0 + 8 * s; };
  auto q_empty = [&](int s) { return bar0 + 8 * (QS + s); };
  auto k_full = [&](int s) { return bar0 + 8 * (2 * QS + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (2 * QS + S + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (2 * QS + 2 * S + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (2 * QS + 3 * S + s); };
  const uint32_t s_full = bar0 + 8 * (2 * QS + 4 * S);  // S and dP in TMEM
  const uint32_t s_free = s_full + 8;                    // ... read by the math warps
  const uint32_t ds_full = s_full + 16;                  // dS in TMEM
  const uint32_t ds_free = s_full + 24;                  // ... read by the dQ MMA
  const uint32_t dq_full = s_full + 32;                  // the unit's dQ complete
  const uint32_t drain_bar = s_full + 40;
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  auto q_tile = [&](int s) { return sbase + Cfg::kOffQ + s * 2 * Cfg::kTileBytes; };
  auto do_tile = [&](int s) { return q_tile(s) + Cfg::kTileBytes; };
  auto k_tile = [&](int s) { return sbase + Cfg::kOffK + s * 2 * Cfg::kTileBytes; };
  auto v_tile = [&](int s) { return k_tile(s) + Cfg::kTileBytes; };
  auto rows_of = [&](int s) { return sbase + Cfg::kOffRow + s * 2 * Cfg::kRowBytes; };

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int s = 0; s < QS; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), 1);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, Cfg::kMathThreads);
    mbar_init(ds_full, Cfg::kMathThreads);
    mbar_init(ds_free, 1);
    mbar_init(dq_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_base_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the set-up above touches shared and tensor memory only; global memory
  // waits for the previous kernel in the stream
  pdl_wait();
  const uint32_t tmem = *tmem_base_slot;
  const int G = gridDim.x;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t q_cnt = 0, kv_cnt = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode<false>(p, u);
        const int qs = q_cnt % QS;
        ok = mbar_wait(q_empty(qs), ((q_cnt / QS) & 1) ^ 1);
        if (!ok) break;
        ++q_cnt;
        // the tile's -LSE2 and -D rows (per-head padded layout of the workspace)
        const long long qrow = (long long)w.bh * p.n_t * kTile + w.i0 * kTile;
        mbar_arrive_expect_tx(q_full(qs), 2 * Cfg::kTileBytes + 2 * Cfg::kRowBytes);
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_3d(q_tile(qs) + bx * 16384, &tm_q, bx * 64, w.i0 * kTile, w.bh, q_full(qs));
          tma_load_3d(do_tile(qs) + bx * 16384, &tm_do, bx * 64, w.i0 * kTile, w.bh, q_full(qs));
        }
        bulk_load(rows_of(qs), dp.lse2 + qrow, Cfg::kRowBytes, q_full(qs));
        bulk_load(rows_of(qs) + Cfg::kRowBytes, dp.delta + qrow, Cfg::kRowBytes, q_full(qs));
        for (int j = fwd_next(p, w, 0); j < w.j_end && ok; j = fwd_next(p, w, j + 1)) {
          const int s = kv_cnt % S;
          const uint32_t ph = (kv_cnt / S) & 1;
          const int krow = j * kTile;  // within head w.bh
          ok = mbar_wait(k_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(k_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(k_tile(s) + bx * 16384, &tm_k, bx * 64, krow, w.bh, k_full(s));
          ok = mbar_wait(v_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(v_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(v_tile(s) + bx * 16384, &tm_v, bx * 64, krow, w.bh, v_full(s));
          ++kv_cnt;
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);  // S, dP (K-major)
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);   // dQ: B = K_j MN-major
      const uint64_t desc_q0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);
      const uint64_t desc_k0 = sw128_desc(sbase + Cfg::kOffK, 16, 1024);
      const uint64_t desc_kmn0 = sw128_desc(sbase + Cfg::kOffK, 16384, 1024);
      uint32_t q_cnt = 0, kv_cnt = 0, sf_cnt = 0, ds_cnt = 0;
      bool s_pending = false;  // an S/dP has been issued whose s_free is not yet awaited
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode<false>(p, u);
        const int qs = q_cnt % QS;
        ok = mbar_wait(q_full(qs), (q_cnt / QS) & 1);
        ++q_cnt;
        if (!ok) break;
        const uint32_t q_off = (q_tile(qs) - (sbase + Cfg::kOffQ)) >> 4;
        const uint32_t do_off = q_off + (Cfg::kTileBytes >> 4);
        // S = Q K^T and dP = dO V^T for ring index c, once the math warps
        // have read the previous S and dP
        auto issue_sdp = [&](uint32_t c) -> bool {
          if (s_pending) {
            if (!mbar_wait(s_free, sf_cnt & 1)) return false;
            ++sf_cnt;
            s_pending = false;
          }
          const int s = c % S;
          if (!mbar_wait(k_full(s), (c / S) & 1) || !mbar_wait(v_full(s), (c / S) & 1))
            return false;
          tc_fence_after();
          const uint32_t k_off = (s * 2 * Cfg::kTileBytes) >> 4;
          const uint32_t v_off = k_off + (Cfg::kTileBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            umma_ss(tmem + Cfg::kColS, desc_q0 + q_off + off, desc_k0 + k_off + off, idesc_s,
                    kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            umma_ss(tmem + Cfg::kColDP, desc_q0 + do_off + off, desc_k0 + v_off + off, idesc_s,
                    kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full);
          umma_commit(v_empty(s));
          s_pending = true;
          return true;
        };
        int j = fwd_next(p, w, 0);
        int k = 0;  // visits of this unit
        if (j < w.j_end) ok = issue_sdp(kv_cnt);
        while (ok && j < w.j_end) {
          const uint32_t c = kv_cnt + k;
          const int j2 = fwd_next(p, w, j + 1);
          if (j2 < w.j_end) {
            ok = issue_sdp(c + 1);
            if (!ok) break;
          }
          // dQ += dS K_j once dS is in TMEM
          ok = mbar_wait(ds_full, ds_cnt & 1);
          ++ds_cnt;
          if (!ok) break;
          tc_fence_after();
          const uint32_t kmn_off = ((c % S) * 2 * Cfg::kTileBytes) >> 4;
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + Cfg::kColDQ, tmem + Cfg::kColDS + kk * 8,
                    desc_kmn0 + kmn_off + ((kk * 2048) >> 4), idesc_dq,
                    (k > 0 || kk > 0) ? 1u : 0u);
          umma_commit(ds_free);
          umma_commit(k_empty(c % S));
          if (j2 >= w.j_end) umma_commit(dq_full);
          j = j2;
          ++k;
          if (*abort_flag) ok = false;
        }
        if (!ok) break;
        umma_commit(q_empty(qs));  // every S and dP of the unit has been issued
        kv_cnt += k;
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ math
    const int hh = (warp - 4) >> 2;  // warpgroup: keys 64 hh .. 64 hh + 63 of each tile
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const float* rows_base = reinterpret_cast<const float*>(smem + Cfg::kOffRow);
    uint32_t q_cnt = 0, s_cnt = 0, ds_cnt = 0, dq_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int u = unit_for_round(round, blockIdx.x, G);
      if (u >= p.num_units) break;
      const FwdUnit w = fwd_decode<false>(p, u);
      const int qs = q_cnt % QS;
      const uint32_t q_par = (q_cnt / QS) & 1;
      ++q_cnt;
      const int row = w.i0 * kTile + r_local;  // query index within the head
      uint4* out_row = reinterpret_cast<uint4*>(dp.dq + ((size_t)w.bh * p.N + row) * D);
      const bool row_ok = row < p.N;  // rows of a partial last tile beyond N: no output
      int j = fwd_next(p, w, 0);
      if (j >= w.j_end) {
        // no key visible to this query tile: dQ = 0 (Q and the rows are not read)
#pragma unroll
        for (int c = hh * D / 16; c < (hh + 1) * D / 16; ++c)
          if (row_ok) out_row[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      // this row's -LSE2 and -D (the slot is refilled only after the unit's
      // last dQ MMA, which follows this warpgroup's last dS)
      ok = __all_sync(0xffffffffu, mbar_wait(q_full(qs), q_par));
      if (!ok) break;
      const float nl = rows_base[qs * 2 * kTile + r_local];
      const float nd = rows_base[qs * 2 * kTile + kTile + r_local];
      const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
      const uint64_t nl2 = f2_pack(nl, nl);
      const uint64_t nd2 = f2_pack(nd, nd);
      for (; j < w.j_end; j = fwd_next(p, w, j + 1)) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, s_cnt & 1));
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();
        const bool diag = p.causal && (j == w.i0);
        const int kv_lim = w.L - j * kTile;  // keys >= kv_lim are padding
        const int lim = diag ? min(r_local + 1, kv_lim) : kv_lim;
        const bool boundary = diag || kv_lim < kTile;
        {
          uint32_t sr[2][32], pr[2][32];
          tmem_ld32(t_lane + Cfg::kColS + hh * 64, sr[0]);
          tmem_ld32(t_lane + Cfg::kColS + hh * 64 + 32, sr[1]);
          tmem_ld32(t_lane + Cfg::kColDP + hh * 64, pr[0]);
          tmem_ld32(t_lane + Cfg::kColDP + hh * 64 + 32, pr[1]);
          tmem_wait_ld();
          reg_fence32(sr[0]);
          reg_fence32(sr[1]);
          reg_fence32(pr[0]);
          reg_fence32(pr[1]);
          // this warpgroup's half of S and dP is in registers: once both halves
          // are, the next S / dP may overwrite them
          tc_fence_before();
          mbar_arrive(s_free);
          if (ds_cnt > 0) {
            // dS is overwritten below: the previous dQ MMA must have read it
            ok = __all_sync(0xffffffffu, mbar_wait(ds_free, (ds_cnt - 1) & 1));
            if (!ok) break;
            tc_fence_after();
          }
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              const int key = hh * 64 + c * 32 + 2 * e;  // key within the tile
              const uint64_t x = f2_fma(f2_pack(__uint_as_float(sr[c][2 * e]),
                                                __uint_as_float(sr[c][2 * e + 1])),
                                        scale2, nl2);
              float x0, x1;
              f2_unpack(x, x0, x1);
              float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              if (boundary) {
                p0 = (key < lim) ? p0 : 0.f;
                p1 = (key + 1 < lim) ? p1 : 0.f;
              }
              const uint64_t t = f2_add(f2_pack(__uint_as_float(pr[c][2 * e]),
                                                __uint_as_float(pr[c][2 * e + 1])),
                                        nd2);
              float d0, d1;
              f2_unpack(f2_mul(t, f2_pack(p0, p1)), d0, d1);
              pk[e] = pack_bf16x2(d0, d1);
            }
            tmem_st16(t_lane + Cfg::kColDS + hh * 32 + c * 16, pk);
          }
        }
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_full);
        ++ds_cnt;
        if (*abort_flag) {
          ok = false;
          break;
        }
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(dq_full, dq_cnt & 1));
      ++dq_cnt;
      if (!ok) break;
      tc_fence_after();
#pragma unroll 1
      for (int c = hh * D / 64; c < (hh + 1) * D / 64; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + Cfg::kColDQ + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * dp.scale,
                              __uint_as_float(r[2 * e + 1]) * dp.scale);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4)
          if (row_ok)
            out_row[c * 4 + v4] =
                make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
      }
      tc_fence_before();
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace fa
