// fa_fwd.cuh - forward kernel: exact attention with an online softmax, tiled
// so that the N x N score matrix never leaves the SM.
//
// Method: "FlashAttention: Fast and Memory-Efficient Exact Attention with
// IO-Awareness" (opendecode.dev summary, "The key idea"): queries, keys and
// values are cut into tiles that fit on chip; for each query row a running
// maximum and running sum are kept and the partial output is rescaled as
// each key/value tile arrives, so the result equals standard attention.
// "FlashAttention, Decoded" ("The Hardware Picture") gives the reason: the
// score tile lives in on-chip memory only.
//
// B200 mapping (one persistent CTA per SM, 12 warps):
//   warp 0      TMA producer: Q tiles of the unit, then the K/V tiles it
//               visits, through a kStages-deep mbarrier ring.
//   warp 1      MMA issuer (one thread): S = Q K^T and O += P V as tcgen05
//               MMAs accumulating in tensor memory.  Also owns the TMEM
//               allocation.
//   warps 4-7   softmax for query tile A (TMEM lanes 0-127, one row each)
//   warps 8-11  softmax for query tile B
// A work unit is (b, h, pair of 128-row query tiles A = 2p, B = 2p+1).  The
// two tiles share every K/V tile load and alternate on the tensor core, so
// one tile's softmax runs while the other tile's MMAs execute.
//
// TMEM columns: S_A [0,128), S_B [128,256), O_A [256,256+D), O_B after it.
// P (bf16) is written over the first 64 columns of its S tile and read from
// there by the P V MMA.  tcgen05 MMAs issued by one thread execute in issue
// order, which makes this aliasing safe: the next S MMA into the same
// columns is issued after the P V MMA that reads them.
//
// Online softmax state per row (thread): m (running max, in units of
// log2, scale folded in), l (running sum).  O is rescaled only when the row
// max grows by more than kRescaleLog2 (a factor of 256); otherwise P is
// formed against the stale max, which keeps P <= 256 and l, O finite in
// float32.  Any reference max gives the same O / l and LSE in exact
// arithmetic, because O and l are always scaled by the same factor.
#pragma once

#include "sm100.cuh"

namespace fa {

constexpr int kTile = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

struct FwdParams {
  uint16_t* o;
  float* lse;
  const uint8_t* block_mask;
  const int32_t* kv_len;
  uint8_t* visited;
  int B, H, N, n_t;
  int num_pairs;
  int num_units;
  int causal;
  float scale_log2;  // scale * log2(e)
};

template <int D>
struct FwdCfg {
  static constexpr int kThreads = 384;
  // registers per thread: 168 at launch (384 x 168 = 64512); the producer /
  // MMA warpgroup gives back 64 each, the two softmax warpgroups take 32 more:
  // 128 x 104 + 256 x 200 = 64512.
  static constexpr uint32_t kRegsLaunch = 168, kRegsLow = 104, kRegsHigh = 200;
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D bf16 tile
  static constexpr int kBoxes = D / 64;             // 64-column TMA boxes per tile
  static constexpr int kStages = (D == 64) ? 4 : 2;
  static constexpr int kOffQ = 0;  // Q_A, Q_B
  static constexpr int kOffK = kOffQ + 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffBar = kOffV + kStages * kTileBytes;
  // barriers: q_full[2], q_empty[2], k_full[S], k_empty[S], v_full[S], v_empty[S],
  //           s_full[2], p_full[2], o_full[2], drain
  static constexpr int kNumBars = 4 + 4 * kStages + 6 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 512;
  __device__ static constexpr uint32_t col_s(int x) { return x ? 128u : 0u; }
  __device__ static constexpr uint32_t col_o(int x) { return x ? 256u + D : 256u; }
};

// Work-unit order: longest units first (for causal masks the last query
// tiles see the most keys), then snake order over CTAs so that the sum of
// lengths per CTA evens out.
__device__ __forceinline__ int unit_for_round(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

struct FwdUnit {
  int bh, b, iA, iB, has_b, L, j_end;
};

__device__ __forceinline__ FwdUnit fwd_decode(const FwdParams& p, int u) {
  FwdUnit w;
  const int BH = p.B * p.H;
  const int rank = u / BH;  // 0 = longest
  w.bh = u - rank * BH;
  w.b = w.bh / p.H;
  const int pair = p.causal ? (p.num_pairs - 1 - rank) : rank;
  w.iA = 2 * pair;
  w.iB = 2 * pair + 1;
  w.has_b = w.iB < p.n_t;
  int L = p.N;
  if (p.kv_len) {
    L = __ldg(p.kv_len + w.b);
    L = L < 0 ? 0 : (L > p.N ? p.N : L);
  }
  w.L = L;
  int j_end = (L + kTile - 1) / kTile;
  if (p.causal) {
    const int last = w.has_b ? w.iB : w.iA;
    j_end = min(j_end, last + 1);
  }
  w.j_end = j_end;
  return w;
}

// Is key tile j visited by query tile i?  (Some (r, c) in the tile pair is
// allowed.)  Causal: j <= i.  Key padding: j*128 < L.  Block mask: nonzero.
__device__ __forceinline__ bool fwd_tile_on(const FwdParams& p, const FwdUnit& w, int i, int j) {
  if (p.causal && j > i) return false;
  if (j * kTile >= w.L) return false;
  if (p.block_mask && __ldg(p.block_mask + (size_t)i * p.n_t + j) == 0) return false;
  return true;
}

__device__ __forceinline__ int fwd_flags(const FwdParams& p, const FwdUnit& w, int j) {
  int f = fwd_tile_on(p, w, w.iA, j) ? 1 : 0;
  if (w.has_b && fwd_tile_on(p, w, w.iB, j)) f |= 2;
  return f;
}

// First visited key tile >= j (or j_end).
__device__ __forceinline__ int fwd_next(const FwdParams& p, const FwdUnit& w, int j, int& flags) {
  for (; j < w.j_end; ++j) {
    flags = fwd_flags(p, w, j);
    if (flags) return j;
  }
  flags = 0;
  return w.j_end;
}

template <int D>
__global__ void __launch_bounds__(FwdCfg<D>::kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using Cfg = FwdCfg<D>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::kOffBar;
  auto q_full = [&](int x) { return bar0 + 8 * x; };
  auto q_empty = [&](int x) { return bar0 + 8 * (2 + x); };
  auto k_full = [&](int s) { return bar0 + 8 * (4 + s); };
  auto k_empty = [&](int s) { return bar0 + 8 * (4 + S + s); };
  auto v_full = [&](int s) { return bar0 + 8 * (4 + 2 * S + s); };
  auto v_empty = [&](int s) { return bar0 + 8 * (4 + 3 * S + s); };
  auto s_full = [&](int x) { return bar0 + 8 * (4 + 4 * S + x); };
  auto p_full = [&](int x) { return bar0 + 8 * (6 + 4 * S + x); };
  auto o_full = [&](int x) { return bar0 + 8 * (8 + 4 * S + x); };
  const uint32_t drain_bar = bar0 + 8 * (10 + 4 * S);
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(q_full(x), 1);
      mbar_init(q_empty(x), 1);
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 128);
      mbar_init(o_full(x), 1);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      mbar_init(k_empty(s), 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_base_slot), Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_base_slot;
  const int G = gridDim.x;
  static_assert(Cfg::kRegsLow * 128 + Cfg::kRegsHigh * 256 <= Cfg::kRegsLaunch * Cfg::kThreads,
                "register split exceeds the launch allocation");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      uint32_t q_cnt[2] = {0, 0};
      uint32_t kv_cnt = 0;
      bool ok = true;
      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode(p, u);
        const int nq = w.has_b ? 2 : 1;
        for (int x = 0; x < nq && ok; ++x) {
          ok = mbar_wait(q_empty(x), (q_cnt[x] & 1) ^ 1);
          if (!ok) break;
          const int row = w.bh * p.N + (x ? w.iB : w.iA) * kTile;
          mbar_arrive_expect_tx(q_full(x), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_2d(sbase + Cfg::kOffQ + x * Cfg::kTileBytes + bx * 16384, &tm_q, bx * 64, row,
                        q_full(x));
          ++q_cnt[x];
        }
        int fl;
        for (int j = fwd_next(p, w, 0, fl); j < w.j_end && ok; j = fwd_next(p, w, j + 1, fl)) {
          const int s = kv_cnt % S;
          const uint32_t ph = (kv_cnt / S) & 1;
          const int row = w.bh * p.N + j * kTile;
          ok = mbar_wait(k_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(k_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_2d(sbase + Cfg::kOffK + s * Cfg::kTileBytes + bx * 16384, &tm_k, bx * 64, row,
                        k_full(s));
          ok = mbar_wait(v_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(v_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_2d(sbase + Cfg::kOffV + s * Cfg::kTileBytes + bx * 16384, &tm_v, bx * 64, row,
                        v_full(s));
          ++kv_cnt;
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      uint32_t q_cnt[2] = {0, 0};
      uint32_t p_cnt[2] = {0, 0};
      uint32_t kv_cnt = 0;
      bool ok = true;

      // Descriptors: one base per tile; the start-address field (bits 0..13,
      // address >> 4) is advanced by adding (byte offset >> 4).  Tiles lie in
      // the first 256 KB of shared memory, so the field never carries over.
      const uint64_t desc_q0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);
      const uint64_t desc_k0 = sw128_desc(sbase + Cfg::kOffK, 16, 1024);
      const uint64_t desc_v0 = sw128_desc(sbase + Cfg::kOffV, 16384, 1024);
      auto issue_s = [&](int x, int s) {
        const uint64_t dq = desc_q0 + ((x * Cfg::kTileBytes) >> 4);
        const uint64_t dk = desc_k0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full(x));
      };
      auto issue_pv = [&](int x, int s, uint32_t acc) {
        const uint64_t dv = desc_v0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          umma_ts(tmem + Cfg::col_o(x), tmem + Cfg::col_s(x) + kk * 8, dv + ((kk * 2048) >> 4),
                  idesc_pv, (kk > 0 || acc) ? 1u : 0u);
        }
      };

      for (int round = 0; ok; ++round) {
        const int u = unit_for_round(round, blockIdx.x, G);
        if (u >= p.num_units) break;
        const FwdUnit w = fwd_decode(p, u);
        const int nq = w.has_b ? 2 : 1;
        for (int x = 0; x < nq && ok; ++x) {
          ok = mbar_wait(q_full(x), q_cnt[x] & 1);
          ++q_cnt[x];
        }
        if (!ok) break;
        tc_fence_after();
        int started[2] = {0, 0};
        int fl = 0;
        int j = fwd_next(p, w, 0, fl);
        if (j < w.j_end) {
          const int s = kv_cnt % S;
          ok = mbar_wait(k_full(s), (kv_cnt / S) & 1);
          if (!ok) break;
          tc_fence_after();
          for (int x = 0; x < 2; ++x)
            if (fl & (1 << x)) {
              issue_s(x, s);
              if (p.visited)
                p.visited[((size_t)w.bh * p.n_t + (x ? w.iB : w.iA)) * p.n_t + j] = 1;
            }
          umma_commit(k_empty(s));
        }
        while (j < w.j_end && ok) {
          const int s = kv_cnt % S;
          int fln = 0;
          const int jn = fwd_next(p, w, j + 1, fln);
          const uint32_t cn = kv_cnt + 1;
          const int sn = cn % S;
          bool v_ready = false, k_next_ready = false;
          for (int x = 0; x < 2 && ok; ++x) {
            if (fl & (1 << x)) {
              ok = mbar_wait(p_full(x), p_cnt[x] & 1);
              ++p_cnt[x];
              if (!ok) break;
              if (!v_ready) {
                ok = mbar_wait(v_full(s), (kv_cnt / S) & 1);
                if (!ok) break;
                v_ready = true;
              }
              tc_fence_after();
              issue_pv(x, s, started[x]);
              started[x] = 1;
            }
            if (x == 1) umma_commit(v_empty(s));
            if (jn < w.j_end && (fln & (1 << x))) {
              if (!k_next_ready) {
                ok = mbar_wait(k_full(sn), (cn / S) & 1);
                if (!ok) break;
                tc_fence_after();
                k_next_ready = true;
              }
              issue_s(x, sn);
              if (p.visited)
                p.visited[((size_t)w.bh * p.n_t + (x ? w.iB : w.iA)) * p.n_t + jn] = 1;
            }
          }
          if (!ok) break;
          if (jn < w.j_end) umma_commit(k_empty(sn));
          kv_cnt = cn;
          j = jn;
          fl = fln;
          if (*abort_flag) ok = false;
        }
        if (!ok) break;
        for (int x = 0; x < nq; ++x) {
          if (started[x]) umma_commit(o_full(x));
          umma_commit(q_empty(x));
        }
      }
      if (!ok) *abort_flag = 1;
      // all issued MMAs complete before TMEM is released
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    setmaxnreg_dec<Cfg::kRegsLow>();  // idle warps of the first warpgroup
  } else {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<Cfg::kRegsHigh>();
    const int x = (warp >= 8) ? 1 : 0;
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;  // row within the query tile = TMEM lane
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = t_lane + Cfg::col_s(x);
    const uint32_t tO = t_lane + Cfg::col_o(x);
    uint32_t s_cnt = 0, o_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      const int u = unit_for_round(round, blockIdx.x, G);
      if (u >= p.num_units) break;
      const FwdUnit w = fwd_decode(p, u);
      if (x == 1 && !w.has_b) continue;
      const int i = x ? w.iB : w.iA;
      const int row = i * kTile + r_local;  // query index within the head
      float m_used = -INFINITY;              // log2 domain, scale folded in
      float l = 0.f;
      int cnt = 0;
      int fl = 0;
      for (int j = fwd_next(p, w, 0, fl); j < w.j_end; j = fwd_next(p, w, j + 1, fl)) {
        if (!(fl & (1 << x))) continue;
        ok = __all_sync(0xffffffffu, mbar_wait(s_full(x), s_cnt & 1));
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();
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
        // element masks on boundary tiles only
        const bool diag = p.causal && (j == i);
        const int kv_lim = w.L - j * kTile;  // keys c >= kv_lim are padding
        if (diag || kv_lim < kTile) {
          const int lim = diag ? min(r_local + 1, kv_lim) : kv_lim;
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            if (c >= lim) sv[c] = -INFINITY;
        }
        float mx = sv[0];
#pragma unroll
        for (int c = 1; c < kTile; ++c) mx = fmaxf(mx, sv[c]);
        const float m_new = mx * p.scale_log2;  // -inf if the whole row is masked here
        float alpha = 1.f;
        bool rescale = false;
        if (cnt == 0) {
          m_used = m_new;
        } else if (m_new > m_used + kRescaleLog2) {
          alpha = ex2_approx(m_used - m_new);  // m_used may be -inf -> 0
          m_used = m_new;
          l *= alpha;
          rescale = true;
        }
        if (__any_sync(0xffffffffu, rescale)) {
          uint32_t r[32];
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tO + c * 32, r);
          }
        }
        const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2_approx(fmaf(sv[c * 32 + 2 * e], p.scale_log2, -m_sub));
            const float p1 = ex2_approx(fmaf(sv[c * 32 + 2 * e + 1], p.scale_log2, -m_sub));
            lsum += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16(tS + c * 16, pk);
        }
        l += lsum;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(x));
        ++cnt;
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) break;
      // ---------------------------------------------------- epilogue
      const size_t grow = (size_t)w.bh * p.N + row;
      uint4* orow = reinterpret_cast<uint4*>(p.o + grow * D);
      if (cnt > 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(o_full(x), o_cnt & 1));
        ++o_cnt;
        if (!ok) break;
        tc_fence_after();
        const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tO + c * 32, r);
          tmem_wait_ld();
          reg_fence32(r);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                __uint_as_float(r[2 * e + 1]) * inv_l);
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            orow[c * 4 + v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
        tc_fence_before();
        p.lse[grow] = (l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
      } else {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) orow[c] = make_uint4(0, 0, 0, 0);
        p.lse[grow] = -INFINITY;
      }
    }
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace fa
