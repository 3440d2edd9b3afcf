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
//   warp 0      TMA producer: takes work units from a counter shared by all
//               CTAs and publishes them to the other roles through a
//               shared-memory ring; loads the unit's Q tile(s) (double-
//               buffered across units where shared memory allows), then the
//               K/V tiles it visits, through a kStages-deep mbarrier ring
//   warp 1      owns the TMEM allocation; issues MMAs (one thread): for both
//               warpgroups at D = 128, for warpgroup 0 at D = 64
//   warp 2      D = 64: issues warpgroup 1's MMAs
//   warps 4-7   softmax warpgroup 0 (TMEM lanes 0-127, one query row each)
//   warps 8-11  softmax warpgroup 1
// A single MMA-issuing thread beside eight busy softmax warps gets too few
// issue slots to keep the tensor core fed, hence one issuer per warpgroup
// where the layout allows it (D = 64).
// Two ways of filling a work unit, chosen per launch:
//  * pair mode (no block mask): the unit is (b, h, query tiles 2p and 2p+1).
//    Both tiles visit the same key tiles (up to the causal diagonal), so
//    every K/V tile is loaded once for 256 query rows; softmax warpgroup x
//    owns query tile 2p+x outright.
//  * split mode (block mask): the unit is (b, h, one query tile), whose
//    visited key tiles are dealt alternately to the two warpgroups; each
//    keeps its own running (m, l) and O, and the two partial results are
//    merged at the end of the unit (the online-softmax rescaling applied
//    once more).  Random masks give two query tiles few key tiles in common,
//    so pairing them would leave one warpgroup idle.
// Either way one warpgroup's softmax runs while the tensor core works for
// the other.
//
// TMEM columns: S_0 [0,128), S_1 [128,256), O_0 [256,256+D), O_1 after it.
// D = 64: P_0 [384,448), P_1 [448,512) (bf16, two per column).  Once all of
// warpgroup x holds S_x in registers (s_free) its issuer issues the next
// S_x, so S_x(j+1) runs while softmax(j) runs; the P V MMA signals p_free
// once it has read P_x.  D = 128: no room for P, which is written over the
// first 64 columns of its S tile; tcgen05 MMAs issued by one thread execute
// in issue order, which makes this aliasing safe: the next S MMA into the
// same columns is issued after the P V MMA that reads them.
//
// Rows of a partial last query tile beyond N are computed (their Q rows
// load as zero) but not stored; keys beyond N are masked like key padding.
//
// Online softmax state per row (thread): m (running max, in units of
// log2, scale folded in), l (running sum).  O is rescaled only when the row
// max grows by more than kRescaleLog2 (a factor of 256); otherwise P is
// formed against the stale max, which keeps P <= 256 and l, O finite in
// float32.  Any reference max gives the same O / l and LSE in exact
// arithmetic, because O and l are always scaled by the same factor.
#pragma once

#include <type_traits>

#include "sm100.cuh"

namespace fa {

constexpr int kTile = 128;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.0f;

// Dropout on P.  Element (head bh, query r, key c) is kept when its 16-bit
// draw is at least t: the draw is value c % 8 of Philox-4x32-10 with counter
// (c / 8, r, bh, offset) and key (seed_lo, seed_hi), value k being the low
// (even k) or high (odd k) half of output word k / 2.  Kept entries weigh
// w = 65536 / (65536 - t), dropped ones 0.
struct DropoutParams {
  uint32_t t_hi;     // t << 16: low half kept iff (word << 16) >= t_hi, high iff word >= t_hi
  float w;
  uint32_t offset;
  uint32_t rk[20];   // the key's round keys, see philox4x32_10_rk
};

// keep bits of one draw's eight values (bit k = value k)
__device__ __forceinline__ uint32_t keep_bits8(const uint4 d, uint32_t t_hi) {
  const uint32_t wd[4] = {d.x, d.y, d.z, d.w};
  uint32_t b = 0;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    b |= static_cast<uint32_t>((wd[v] << 16) >= t_hi) << (2 * v);
    b |= static_cast<uint32_t>(wd[v] >= t_hi) << (2 * v + 1);
  }
  return b;
}

// Packed variable-length batches: sequence b holds tokens cu_seqlens[b] ..
// cu_seqlens[b+1] - 1 of [T][H][d] tensors.  The values are clamped so that
// every row index stays inside [0, T): the start into [0, T], the length into
// [0, min(N, T - start)] (N = the longest sequence, the unit grid's size).
struct SeqSpan {
  int start, len;
};
__device__ __forceinline__ SeqSpan seq_span(const int32_t* cu, int b, int N, int T) {
  const long long s = min(max(static_cast<long long>(__ldg(cu + b)), 0ll), static_cast<long long>(T));
  const long long len = static_cast<long long>(__ldg(cu + b + 1)) - s;
  const long long cap = min(static_cast<long long>(N), static_cast<long long>(T) - s);
  return {static_cast<int>(s), static_cast<int>(max(0ll, min(len, cap)))};
}

// A 128-row tile of one head: [B*H][N][d] tensors are mapped as (d, N, B*H)
// and packed [T][H][d] tensors as (d, H, T) (strides increasing in both), so
// the tile's (row, head) are the map's (y, z), or (z, y) when packed.
__device__ __forceinline__ int2 tile_yz(bool packed, int row, int head) {
  return packed ? make_int2(head, row) : make_int2(row, head);
}

struct FwdParams {
  uint16_t* o;
  float* lse;
  const uint8_t* block_mask;
  const int32_t* kv_len;
  uint8_t* visited;
  // packed variable-length batches (null: the [B][H][N][d] layout); N is then
  // the longest sequence and T the number of tokens
  const int32_t* cu_seqlens;
  int T;
  long long o_stride;  // elements between consecutive rows of one head's O (d, or H*d packed)
  int dcols;           // the tensors' head dimension d (<= D; columns D > d read as zeros)
  int B, H, N, n_t;
  int num_units;
  int heads_per_group;  // unit order: see fwd_decode
  int causal;
  float scale_log2;  // scale * log2(e)
  int counter_slot;  // this launch's work counter: g_fwd_work[counter_slot]
  DropoutParams drop;  // read by kernels instantiated with kDrop only
};

// Work counters of the forward kernel, which has no workspace.  Launch t uses
// slot t % kFwdCounterSlots (the host hands the slots out in turn): its CTAs
// take units with atomicAdd on word 0 and count themselves out on word 1; the
// last CTA to finish sets both back to zero for the launch that reuses the
// slot.  Launches that are in flight together on one device (other streams)
// therefore use different slots as long as fewer than kFwdCounterSlots of
// them overlap.
constexpr int kFwdCounterSlots = 1024;
static __device__ unsigned int g_fwd_work[kFwdCounterSlots][2];

// Called by one thread of each CTA once the CTA takes no more units: the last
// CTA of the launch to get here sets the slot back to zero.
__device__ __forceinline__ void fwd_count_out(int slot) {
  __threadfence();
  if (atomicAdd(&g_fwd_work[slot][1], 1u) == gridDim.x - 1) {
    atomicExch(&g_fwd_work[slot][0], 0u);
    atomicExch(&g_fwd_work[slot][1], 0u);
  }
}

// Unit records: the producer takes each work unit from the launch's counter
// and publishes its index in a ring of kUnitRing shared-memory slots for the
// other roles; -1 marks the end of the work.
constexpr int kUnitRing = 4;

template <int D, bool kPair>
struct FwdCfg {
  static constexpr int kThreads = 384;
  // registers per thread: 168 at launch (384 x 168 = 64512); the producer /
  // MMA warpgroup gives back 64 each, the two softmax warpgroups take 32 more:
  // 128 x 104 + 256 x 200 = 64512.
  static constexpr uint32_t kRegsLaunch = 168, kRegsLow = 104, kRegsHigh = 200;
  static constexpr int kTileBytes = kTile * D * 2;  // one 128 x D bf16 tile
  static constexpr int kBoxes = D / 64;             // 64-column TMA boxes per tile
  static constexpr int kStages = (D == 64) ? 5 : 2;
  // Q slots: one per unit in flight (double-buffered across units except for
  // pair mode at D = 128, where shared memory holds only one); a slot holds
  // one query tile (split) or two (pair)
  static constexpr int kQPerSlot = kPair ? 2 : 1;
  static constexpr int kQSlots = (kPair && D == 128) ? 1 : 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQSlots * kQPerSlot * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffML = kOffV + kStages * kTileBytes;  // [2 warpgroups][128 rows] (m, l)
  static constexpr int kOffBar = kOffML + 2 * kTile * 8;
  // barriers: q_full[2], q_empty[2], k_full[S], k_empty[S], v_full[S], v_empty[S],
  //           s_full[2], p_full[2], o_full[2], drain[2], ml_ready, merged, s_free[2],
  //           p_free[2], unit_full[R], unit_empty[R]
  static constexpr int kNumBars = 18 + 4 * kStages + 2 * kUnitRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // misc: TMEM base address, abort flag, then the unit ring (kUnitRing ints)
  static constexpr int kOffRing = kOffMisc + 16;
  static constexpr int kSmemBytes = kOffRing + 4 * kUnitRing;
  static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  // pairs (of every 8) whose exponentials ex2_poly2 computes on interior tiles.
  // D = 64 runs both warpgroups' softmax at once, sharing the MUFU unit: a
  // quarter on the FMA pipe balances the two.  At D = 128 the warpgroups take
  // turns and the FMA pipe is the busier one: every exponential goes to MUFU.
  static constexpr int kPolyPer8 = (D == 64) ? 2 : 0;
  // D = 64 leaves 128 TMEM columns after S_0, S_1, O_0, O_1: P gets its own
  // 64 columns per warpgroup, so the next S can be issued as soon as the
  // softmax has read the current one, and each warpgroup has its own MMA
  // issuer.  D = 128 fills TMEM with S and O; P is then written over the first
  // 64 columns of its S tile and one thread issues all MMAs.
  static constexpr bool kSepP = (D == 64);
  __device__ static constexpr uint32_t col_s(int x) { return x ? 128u : 0u; }
  __device__ static constexpr uint32_t col_o(int x) { return x ? 256u + D : 256u; }
  __device__ static constexpr uint32_t col_p(int x) { return kSepP ? 384u + 64u * x : col_s(x); }
  // Pair mode at D = 64: a warpgroup stages its O tile (bf16, 128-byte
  // swizzled rows) in its own query tile's shared memory, which the unit's
  // S MMAs have finished reading, and one thread writes it with a TMA store;
  // the Q slot is released (q_empty) only after the store has read it.
  static constexpr bool kEpiTma = kSepP && kPair;
};

// Work-unit order: heads are taken in groups whose K and V fit in a share of
// L2 (the units running at the same time then re-read K and V from L2, not
// HBM); inside a group the longest units come first (for causal masks the
// last query tiles see the most keys).  The forward kernel takes units in that
// order from a counter shared by its CTAs; the ordered dQ kernel deals them to
// CTAs in snake order instead (unit_for_round), so that the sum of lengths
// per CTA evens out.
__device__ __forceinline__ int unit_for_round(int round, int cta, int G) {
  return round * G + ((round & 1) ? (G - 1 - cta) : cta);
}

struct FwdUnit {
  int bh, b;
  int nq;        // query rows (N, or the sequence's length)
  int tok_base;  // first row of this head: B*H*N rows (b*H+h)*N, or the sequence's first token
  int tz;        // the head's TMA coordinate: b*H+h, or h (packed)
  bool empty;    // packed: the unit's query tiles lie beyond its sequence
  int i0, i1;           // query tile of warpgroup 0 / 1 (split mode: the same tile)
  int has1;             // pair mode: query tile i1 exists
  int L;                // keys c < L are not padding
  int j_end0, j_end1;   // key tiles below j_end_x may hold an allowed key for tile i_x
  int j_end;            // the unit's key tiles lie below j_end
};

// Unit u -> (head group g, rank within the group, head): ranks are
// interleaved over the group's heads, rank 0 (longest) first.
__device__ __forceinline__ void group_order(int u, int n_t, int BH, int G, int& bh, int& rank) {
  const int per_group = G * n_t;
  const int g = u / per_group;
  const int r = u - g * per_group;
  const int h0 = g * G;
  const int gh = min(G, BH - h0);
  rank = r / gh;
  bh = h0 + (r - rank * gh);
}

template <bool kPair, bool kPacked = false>
__device__ __forceinline__ FwdUnit fwd_decode(const FwdParams& p, int u) {
  FwdUnit w;
  const int per_head = kPair ? (p.n_t + 1) / 2 : p.n_t;
  int rank;  // 0 = longest
  group_order(u, per_head, p.B * p.H, p.heads_per_group, w.bh, rank);
  w.b = w.bh / p.H;
  const int slot = p.causal ? (per_head - 1 - rank) : rank;
  int L = p.N;
  int n_tq = p.n_t;  // query tiles of this head
  if constexpr (kPacked) {
    const SeqSpan sp = seq_span(p.cu_seqlens, w.b, p.N, p.T);
    const int h = w.bh - w.b * p.H;
    L = sp.len;
    n_tq = (sp.len + kTile - 1) / kTile;
    w.nq = sp.len;
    w.tok_base = sp.start;
    w.tz = h;
  } else {
    if (p.kv_len) {
      L = __ldg(p.kv_len + w.b);
      L = L < 0 ? 0 : (L > p.N ? p.N : L);
    }
    w.nq = p.N;
    w.tok_base = w.bh * p.N;
    w.tz = w.bh;
  }
  w.L = L;
  const int j_kv = (L + kTile - 1) / kTile;  // key tiles holding a key c < L
  if (kPair) {
    w.i0 = 2 * slot;
    w.i1 = 2 * slot + 1;
    w.has1 = w.i1 < n_tq;
  } else {
    w.i0 = w.i1 = slot;
    w.has1 = 0;
  }
  w.empty = w.i0 >= n_tq;
  w.j_end0 = p.causal ? min(j_kv, w.i0 + 1) : j_kv;
  w.j_end1 = (kPair && !w.has1) ? 0 : (p.causal ? min(j_kv, w.i1 + 1) : j_kv);
  w.j_end = max(w.j_end0, w.j_end1);
  return w;
}

// Split mode: first key tile >= j that query tile w.i0 visits (or j_end):
// tiles below j_end hold an allowed key for causal and key-padding masks; the
// block mask is the only test left.  (Pair mode has no block mask: its tiles
// are all of [0, j_end_x).)
__device__ __forceinline__ int fwd_next(const FwdParams& p, const FwdUnit& w, int j) {
  if (!p.block_mask) return j < w.j_end ? j : w.j_end;
  const uint8_t* row = p.block_mask + (size_t)w.i0 * p.n_t;
  for (; j < w.j_end; ++j)
    if (__ldg(row + j)) return j;
  return w.j_end;
}

template <int D, bool kPair, bool kDrop = false, bool kPacked = false>
__global__ void __launch_bounds__(FwdCfg<D, kPair>::kThreads, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                  const FwdParams p) {
  using Cfg = FwdCfg<D, kPair>;
  constexpr int S = Cfg::kStages;
  constexpr int QSLOTS = Cfg::kQSlots;
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_launch_dependents();
  if (!smem_aligned_1024(smem)) {
    if (threadIdx.x == 0) fwd_count_out(p.counter_slot);
    return;
  }
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
  auto drain = [&](int x) { return x ? bar0 + 8 * (17 + 4 * S) : drain_bar; };
  // split mode: the two softmax warpgroups meet twice per unit in the merge:
  // (m, l) published, and both partial outputs read (bounded waits, 256 arrivals)
  const uint32_t ml_ready = bar0 + 8 * (11 + 4 * S);
  const uint32_t merged = bar0 + 8 * (12 + 4 * S);
  // separate-P layout: warpgroup x has read S_x (128 arrivals) / P V_x has read P_x
  auto s_free = [&](int x) { return bar0 + 8 * (13 + 4 * S + x); };
  auto p_free = [&](int x) { return bar0 + 8 * (15 + 4 * S + x); };
  constexpr int UR = kUnitRing;
  auto unit_full = [&](int r) { return bar0 + 8 * (18 + 4 * S + r); };
  auto unit_empty = [&](int r) { return bar0 + 8 * (18 + 4 * S + UR + r); };
  static_assert(Cfg::kNumBars == 18 + 4 * S + 2 * UR, "barrier layout");
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  volatile int* unit_ring = reinterpret_cast<volatile int*>(smem + Cfg::kOffRing);
  // the warps that read every unit record: the MMA issuer(s) and 8 softmax warps
  constexpr uint32_t kUnitReaders = (Cfg::kSepP ? 2 : 1) + 8;
  // one thread's read of round r's record (it releases the slot)
  auto fetch_one = [&](int r, int& u) -> bool {
    const int sl = r % UR;
    if (!mbar_wait(unit_full(sl), (r / UR) & 1)) return false;
    u = unit_ring[sl];
    mbar_arrive(unit_empty(sl));
    return true;
  };
  // a whole warp's read (lane 0 releases the slot)
  auto fetch_warp = [&](int r, int& u) -> bool {
    const int sl = r % UR;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(unit_full(sl), (r / UR) & 1));
    if (ok) u = unit_ring[sl];
    __syncwarp();
    if (ok && lane_id() == 0) mbar_arrive(unit_empty(sl));
    return ok;
  };
  float2* ml_smem = reinterpret_cast<float2*>(smem + Cfg::kOffML);  // [2][128] (m, l)
  // shared-memory address of query tile x (0 / 1) of Q slot q
  auto q_tile = [&](int q, int x) {
    return sbase + Cfg::kOffQ + (q * Cfg::kQPerSlot + (kPair ? x : 0)) * Cfg::kTileBytes;
  };

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(q_full(x), 1);
      // separate-P layout: both warpgroups' issuers arrive
      mbar_init(q_empty(x), (Cfg::kSepP ? 2 : 1) + (Cfg::kEpiTma ? 2 : 0));
      mbar_init(s_full(x), 1);
      mbar_init(p_full(x), 128);
      mbar_init(o_full(x), 1);
      mbar_init(s_free(x), 128);
      mbar_init(p_free(x), 1);
    }
    for (int s = 0; s < S; ++s) {
      mbar_init(k_full(s), 1);
      // separate-P pair mode: both issuers arrive for every tile of the unit
      mbar_init(k_empty(s), (Cfg::kSepP && kPair) ? 2 : 1);
      mbar_init(v_full(s), 1);
      mbar_init(v_empty(s), (Cfg::kSepP && kPair) ? 2 : 1);
    }
    mbar_init(drain_bar, 1);
    mbar_init(drain(1), 1);
    mbar_init(ml_ready, 256);
    mbar_init(merged, 256);
    for (int r = 0; r < UR; ++r) {
      mbar_init(unit_full(r), 1);
      mbar_init(unit_empty(r), kUnitReaders);
    }
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    if (Cfg::kEpiTma) prefetch_tmap(&tm_o);
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
  static_assert(Cfg::kRegsLow * 128 + Cfg::kRegsHigh * 256 <= Cfg::kRegsLaunch * Cfg::kThreads,
                "register split exceeds the launch allocation");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      uint32_t q_cnt = 0, kv_cnt = 0;
      bool ok = true;
      // Units come from the launch's counter, shared by all CTAs, in the order
      // fwd_decode gives them (longest first within each head group), so that
      // the CTAs finish together whatever the unit lengths.  Records are
      // published one round ahead (the issuers read the next unit's record at
      // the end of this one); after the work runs out, one record marks the end.
      unsigned int* const work_next = &g_fwd_work[p.counter_slot][0];
      int published = 0;
      bool ended = false;
      auto publish_through = [&](int upto) -> bool {
        while (!ended && published <= upto) {
          int un = static_cast<int>(atomicAdd(work_next, 1u));
          if (un >= p.num_units) {
            un = -1;
          } else if (kPacked && fwd_decode<kPair, kPacked>(p, un).empty) {
            continue;  // query tiles past a shorter sequence's end: no work
          }
          const int sl = published % UR;
          if (!mbar_wait(unit_empty(sl), ((published / UR) & 1) ^ 1)) return false;
          unit_ring[sl] = un;
          mbar_arrive(unit_full(sl));
          ++published;
          if (un < 0) ended = true;
        }
        return true;
      };
      for (int round = 0; ok; ++round) {
        ok = publish_through(round + 1);
        if (!ok) break;
        const int u = unit_ring[round % UR];
        if (u < 0) break;
        const FwdUnit w = fwd_decode<kPair, kPacked>(p, u);
        const int qs = q_cnt % QSLOTS;
        ok = mbar_wait(q_empty(qs), ((q_cnt / QSLOTS) & 1) ^ 1);
        if (!ok) break;
        ++q_cnt;
        const int nq = (kPair && w.has1) ? 2 : 1;
        mbar_arrive_expect_tx(q_full(qs), nq * Cfg::kTileBytes);
        for (int x = 0; x < nq; ++x) {
          const int2 yz =
              tile_yz(kPacked, (kPacked ? w.tok_base : 0) + (x ? w.i1 : w.i0) * kTile, w.tz);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(q_tile(qs, x) + bx * 16384, &tm_q, bx * 64, yz.x, yz.y, q_full(qs));
        }
        for (int j = fwd_next(p, w, 0); j < w.j_end && ok; j = fwd_next(p, w, j + 1)) {
          const int s = kv_cnt % S;
          const uint32_t ph = (kv_cnt / S) & 1;
          // packed batches: rows past the sequence's end belong to the next
          // sequence; they are masked (keys) or not stored (queries)
          const int2 yz =
              tile_yz(kPacked, (kPacked ? w.tok_base : 0) + j * kTile, w.tz);
          ok = mbar_wait(k_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(k_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(sbase + Cfg::kOffK + s * Cfg::kTileBytes + bx * 16384, &tm_k, bx * 64,
                        yz.x, yz.y, k_full(s));
          ok = mbar_wait(v_empty(s), ph ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(v_full(s), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(sbase + Cfg::kOffV + s * Cfg::kTileBytes + bx * 16384, &tm_v, bx * 64,
                        yz.x, yz.y, v_full(s));
          ++kv_cnt;
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1 && !Cfg::kSepP) {
    // ------------------------------------------------- MMA issuer (D = 128)
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      // Descriptors: one base per operand; the start-address field (bits 0..13,
      // address >> 4) is advanced by adding (byte offset >> 4).  Tiles lie in
      // the first 256 KB of shared memory, so the field never carries over.
      const uint64_t desc_q0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);
      const uint64_t desc_k0 = sw128_desc(sbase + Cfg::kOffK, 16, 1024);
      const uint64_t desc_v0 = sw128_desc(sbase + Cfg::kOffV, 16384, 1024);
      uint32_t q_cnt = 0, kv_cnt = 0;
      uint32_t p_cnt[2] = {0, 0};
      bool ok = true;
      // Pair mode with two Q slots looks one unit ahead: warpgroup x's first S
      // of the next unit is issued right after its last P V of this one, so
      // its epilogue overlaps that MMA and the one-step offset between the two
      // warpgroups carries over from unit to unit.
      constexpr bool kLook = kPair && QSLOTS == 2;
      uint32_t pre = 0;      // bit x: S_x of this unit's first key tile already issued
      bool pre_q = false;    // this unit's Q already waited for
      bool pre_k = false;    // this unit's first K tile already waited for
      int u_ahead = -2;      // the next round's record when already read (-2: not read)
      for (int round = 0; ok; ++round) {
        int u = u_ahead;
        u_ahead = -2;
        if (u == -2 && !fetch_one(round, u)) {
          ok = false;
          break;
        }
        if (u < 0) break;
        const FwdUnit w = fwd_decode<kPair, kPacked>(p, u);
        const int qs = q_cnt % QSLOTS;
        if (!pre_q) ok = mbar_wait(q_full(qs), (q_cnt / QSLOTS) & 1);
        ++q_cnt;
        if (!ok) break;
        // S_x = Q_x K^T of unit w's key tile j, Q from slot q, K from stage c % S,
        // into warpgroup x's S columns
        auto issue_s_of = [&](const FwdUnit& wu, int q, int x, uint32_t c, int j) {
          const int s = c % S;
          const uint64_t dq = desc_q0 + ((q_tile(q, x) - (sbase + Cfg::kOffQ)) >> 4);
          const uint64_t dk = desc_k0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
            umma_ss(tmem + Cfg::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
          }
          umma_commit(s_full(x));
          if (p.visited)
            p.visited[((size_t)wu.bh * p.n_t + (x ? wu.i1 : wu.i0)) * p.n_t + j] = 1;
        };
        auto issue_s = [&](int x, uint32_t c, int j) { issue_s_of(w, qs, x, c, j); };
        // O_x += P_x V for the stage c % S
        auto issue_pv = [&](int x, uint32_t c, uint32_t acc) {
          const int s = c % S;
          const uint64_t dv = desc_v0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + Cfg::col_o(x), tmem + Cfg::col_s(x) + kk * 8, dv + ((kk * 2048) >> 4),
                    idesc_pv, (kk > 0 || acc) ? 1u : 0u);
        };
        int n_items = 0;  // key tiles consumed by this unit
        if constexpr (kPair) {
          // Both tiles walk key tiles 0 .. j_end - 1; tile x takes those below
          // j_end_x (j_end_0 >= 1 whenever j_end >= 1).  Per key tile: PV_0,
          // S_0(next), PV_1, S_1(next), so that each warpgroup's next S follows
          // its own P V immediately.  In the first unit warpgroup 1 starts one
          // step behind warpgroup 0 (its first S is issued after P V_0(0)), so
          // that one warpgroup's softmax overlaps the other's MMAs instead of
          // competing with it for issue slots.
          const int j_end = w.j_end;
          // the next unit (look-ahead)
          int un = -1;
          if (kLook) {
            if (!fetch_one(round + 1, un)) {
              ok = false;
              break;
            }
            u_ahead = un;
          }
          const bool has_next = kLook && un >= 0;
          FwdUnit wn = w;
          if (has_next) wn = fwd_decode<kPair, kPacked>(p, un);
          const int qsn = q_cnt % QSLOTS;
          const uint32_t cn = kv_cnt + j_end;  // ring index of the next unit's first tile
          uint32_t pre_next = 0;
          bool q_next = false, k_next0 = false;
          if (j_end > 0 && !(pre & 1)) {
            if (!pre_k) ok = mbar_wait(k_full(kv_cnt % S), (kv_cnt / S) & 1);
            if (ok) {
              tc_fence_after();
              issue_s(0, kv_cnt, 0);
            }
          }
          for (int j = 0; j < j_end && ok; ++j) {
            const uint32_t c = kv_cnt + j;
            const bool next = j + 1 < j_end;
            bool v_ready = false, k_next = false;
            for (int x = 0; x < 2 && ok; ++x) {
              const int je = x ? w.j_end1 : w.j_end0;
              if (j < je) {
                ok = mbar_wait(p_full(x), p_cnt[x] & 1);
                ++p_cnt[x];
                if (!ok) break;
                if (!v_ready) {
                  ok = mbar_wait(v_full(c % S), (c / S) & 1);
                  if (!ok) break;
                  v_ready = true;
                }
                tc_fence_after();
                issue_pv(x, c, j > 0);
                if (j == je - 1) umma_commit(o_full(x));
              }
              if (x == 1) umma_commit(v_empty(c % S));
              if (next && j + 1 < je) {
                if (!k_next) {
                  ok = mbar_wait(k_full((c + 1) % S), ((c + 1) / S) & 1);
                  if (!ok) break;
                  tc_fence_after();
                  k_next = true;
                }
                issue_s(x, c + 1, j + 1);
              } else if (has_next && j == je - 1 && (x ? wn.j_end1 : wn.j_end0) > 0) {
                // warpgroup x is done with this unit: its first S of the next one
                if (!q_next) {
                  ok = mbar_wait(q_full(qsn), (q_cnt / QSLOTS) & 1);
                  if (!ok) break;
                  q_next = true;
                }
                if (!k_next0) {
                  ok = mbar_wait(k_full(cn % S), (cn / S) & 1);
                  if (!ok) break;
                  k_next0 = true;
                }
                tc_fence_after();
                issue_s_of(wn, qsn, x, cn, 0);
                pre_next |= 1u << x;
              }
              if (x == 0 && j == 0) {
                // warpgroup 1's first S of this unit, unless issued already;
                // then K of tile 0 has both its readers
                if (w.j_end1 > 0 && !(pre & 2)) issue_s(1, c, 0);
                umma_commit(k_empty(c % S));
              }
            }
            if (ok && next) umma_commit(k_empty((c + 1) % S));
            if (*abort_flag) ok = false;
          }
          if (!ok) break;
          n_items = j_end;
          pre = pre_next;
          pre_q = q_next;
          pre_k = k_next0;
        } else {
          // k-th visited key tile goes to warpgroup k & 1: S(0) first, then per
          // k: P V(k), S(k + 2) (same warpgroup, its S columns are free once
          // P V(k) has read P(k) - tcgen05 MMAs execute in issue order), with
          // S(1) issued right after P V(0)
          auto issue_s_k = [&](int k, int j) -> bool {
            const uint32_t c = kv_cnt + k;
            if (!mbar_wait(k_full(c % S), (c / S) & 1)) return false;
            tc_fence_after();
            issue_s(k & 1, c, j);
            umma_commit(k_empty(c % S));
            return true;
          };
          int jk = fwd_next(p, w, 0);                                   // tile of visit k
          int jk1 = (jk < w.j_end) ? fwd_next(p, w, jk + 1) : w.j_end;  // visit k + 1
          // warpgroup 1's first S (visit 1) is issued after P V(0): see pair mode
          if (jk < w.j_end) ok = issue_s_k(0, jk);
          int k = 0;
          while (ok && jk < w.j_end) {
            const int x = k & 1;
            const uint32_t c = kv_cnt + k;
            const int jk2 = (jk1 < w.j_end) ? fwd_next(p, w, jk1 + 1) : w.j_end;
            ok = mbar_wait(p_full(x), p_cnt[x] & 1);
            ++p_cnt[x];
            if (!ok) break;
            ok = mbar_wait(v_full(c % S), (c / S) & 1);
            if (!ok) break;
            tc_fence_after();
            issue_pv(x, c, k >= 2);
            umma_commit(v_empty(c % S));
            if (k == 0 && jk1 < w.j_end) ok = issue_s_k(1, jk1);
            if (ok && jk2 < w.j_end) ok = issue_s_k(k + 2, jk2);
            jk = jk1;
            jk1 = jk2;
            ++k;
            if (*abort_flag) ok = false;
          }
          if (!ok) break;
          n_items = k;
          if (k >= 1) umma_commit(o_full(0));
          if (k >= 2) umma_commit(o_full(1));
        }
        umma_commit(q_empty(qs));
        kv_cnt += n_items;
      }
      if (!ok) *abort_flag = 1;
      // all issued MMAs complete before TMEM is released
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (Cfg::kSepP && (warp == 1 || warp == 2)) {
    // -------------------------- MMA issuers, one per softmax warpgroup (D = 64)
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      const int x = warp - 1;  // the warpgroup this thread issues for
      // pair mode with two Q slots: the warpgroup's first S of the next unit is
      // issued right after its last S of this one, so its epilogue overlaps it
      constexpr bool kLook = kPair && QSLOTS == 2;
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, 0, 1);
      const uint64_t desc_q0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);
      const uint64_t desc_k0 = sw128_desc(sbase + Cfg::kOffK, 16, 1024);
      const uint64_t desc_v0 = sw128_desc(sbase + Cfg::kOffV, 16384, 1024);
      // S_x = Q (slot q) K^T, K from ring index c; the k_empty commit releases K
      auto issue_s = [&](int q, uint32_t c) {
        const int s = c % S;
        const uint64_t dq = desc_q0 + ((q_tile(q, x) - (sbase + Cfg::kOffQ)) >> 4);
        const uint64_t dk = desc_k0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::col_s(x), dq + off, dk + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full(x));
        umma_commit(k_empty(s));
      };
      // O_x (+)= P_x V, V from ring index c; p_free and v_empty release P_x and V
      auto issue_pv = [&](uint32_t c, uint32_t acc) {
        const int s = c % S;
        const uint64_t dv = desc_v0 + ((s * Cfg::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_ts(tmem + Cfg::col_o(x), tmem + Cfg::col_p(x) + kk * 8, dv + ((kk * 2048) >> 4),
                  idesc_pv, (kk > 0 || acc) ? 1u : 0u);
        umma_commit(p_free(x));
        umma_commit(v_empty(s));
      };
      auto mark = [&](const FwdUnit& wu, int j) {
        if (p.visited) p.visited[((size_t)wu.bh * p.n_t + (x ? wu.i1 : wu.i0)) * p.n_t + j] = 1;
      };
      // Own visits of a unit.  Pair mode: key tiles 0 .. je - 1, ring index =
      // unit base + tile.  Split mode: visits k = x, x + 2, ... of the unit's
      // visited key tiles, ring index = unit base + k.  nvis counts the unit's
      // visits (both warpgroups) seen so far; after the last own visit it is
      // the unit's total.
      auto own_first = [&](const FwdUnit& wu, int& j, int& nvis) {
        if constexpr (kPair) {
          j = 0;
          nvis = 0;
        } else {
          j = fwd_next(p, wu, 0);
          nvis = (j < wu.j_end) ? 1 : 0;
          if (x == 1 && j < wu.j_end) {
            j = fwd_next(p, wu, j + 1);
            nvis += (j < wu.j_end) ? 1 : 0;
          }
        }
      };
      auto own_next = [&](const FwdUnit& wu, int j, int& nvis) -> int {
        if constexpr (kPair) {
          return j + 1;
        } else {
          const int j1 = fwd_next(p, wu, j + 1);  // the other warpgroup's visit
          if (j1 >= wu.j_end) return wu.j_end;
          ++nvis;
          const int j2 = fwd_next(p, wu, j1 + 1);
          if (j2 < wu.j_end) ++nvis;
          return j2;
        }
      };
      uint32_t q_cnt = 0, kv_cnt = 0;  // units started; ring index of the unit's first tile
      uint32_t t_cnt = 0;              // tiles of this warpgroup (s_free / p_full phases)
      bool pre = false;                // this unit's Q awaited and first own S issued
      bool ok = true;
      int u_ahead = -2;  // the next round's record when already read (-2: not read)
      for (int round = 0; ok; ++round) {
        int u = u_ahead;
        u_ahead = -2;
        if (u == -2 && !fetch_one(round, u)) {
          ok = false;
          break;
        }
        if (u < 0) break;
        const FwdUnit w = fwd_decode<kPair, kPacked>(p, u);
        const int qs = q_cnt % QSLOTS;
        const uint32_t q_par = (q_cnt / QSLOTS) & 1;
        ++q_cnt;
        const int je = kPair ? (x ? w.j_end1 : w.j_end0) : w.j_end;  // own visits lie below je
        int nvis = 0, j = 0;
        own_first(w, j, nvis);
        bool pre_next = false;
        // Q is awaited even without an own visit, so that the q_empty arrival
        // cannot complete the slot's previous phase
        if (!pre) ok = mbar_wait(q_full(qs), q_par);
        if (ok && j < je && !pre) {
          const uint32_t c = kv_cnt + (kPair ? j : x);
          ok = mbar_wait(k_full(c % S), (c / S) & 1);
          if (ok) {
            tc_fence_after();
            issue_s(qs, c);
            mark(w, j);
          }
        }
        if (ok && j >= je) umma_commit(q_empty(qs));  // no own visit: done with Q
        if (!ok) break;
        int cnt = 0;
        while (j < je) {
          const uint32_t c = kv_cnt + (kPair ? j : x + 2 * cnt);
          const int j2 = own_next(w, j, nvis);
          const uint32_t c2 = kv_cnt + (kPair ? j2 : x + 2 * (cnt + 1));
          // the warpgroup has S(j) in registers: the next S
          ok = mbar_wait(s_free(x), t_cnt & 1);
          if (!ok) break;
          if (j2 < je) {
            ok = mbar_wait(k_full(c2 % S), (c2 / S) & 1);
            if (!ok) break;
            tc_fence_after();
            issue_s(qs, c2);
            mark(w, j2);
          } else {
            umma_commit(q_empty(qs));  // this warpgroup's last S on this Q is issued
            if constexpr (kLook) {
              int un = -1;
              if (!fetch_one(round + 1, un)) {
                ok = false;
                break;
              }
              u_ahead = un;
              if (un >= 0) {
                const FwdUnit wn = fwd_decode<kPair, kPacked>(p, un);
                if ((x ? wn.j_end1 : wn.j_end0) > 0) {
                  const int qsn = q_cnt % QSLOTS;
                  const uint32_t cn = kv_cnt + w.j_end;
                  ok = mbar_wait(q_full(qsn), (q_cnt / QSLOTS) & 1) &&
                       mbar_wait(k_full(cn % S), (cn / S) & 1);
                  if (!ok) break;
                  tc_fence_after();
                  issue_s(qsn, cn);
                  mark(wn, 0);
                  pre_next = true;
                }
              }
            }
          }
          // P(j) is in TMEM: O += P V
          ok = mbar_wait(p_full(x), t_cnt & 1) && mbar_wait(v_full(c % S), (c / S) & 1);
          if (!ok) break;
          tc_fence_after();
          issue_pv(c, cnt > 0 ? 1u : 0u);
          if (j2 >= je) umma_commit(o_full(x));
          ++t_cnt;
          ++cnt;
          j = j2;
          if (*abort_flag) {
            ok = false;
            break;
          }
        }
        if (!ok) break;
        // pair mode: the unit's key tiles this warpgroup does not read (the last
        // one of the even query tile under a causal mask; all of them for a
        // missing odd tile): arrive for them on the ring, each after its load
        // has landed, so that the arrival counts for this use of the stage
        if constexpr (kPair) {
          for (int jj = je; jj < w.j_end && ok; ++jj) {
            const uint32_t cc = kv_cnt + jj;
            ok = mbar_wait(k_full(cc % S), (cc / S) & 1) && mbar_wait(v_full(cc % S), (cc / S) & 1);
            if (ok) {
              umma_commit(k_empty(cc % S));
              umma_commit(v_empty(cc % S));
            }
          }
          if (!ok) break;
        }
        kv_cnt += kPair ? w.j_end : nvis;
        pre = pre_next;
      }
      if (!ok) *abort_flag = 1;
      // all issued MMAs complete before TMEM is released
      umma_commit(drain(x));
      mbar_wait(drain(x), 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    setmaxnreg_dec<Cfg::kRegsLow>();  // idle warps of the first warpgroup
  } else {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<Cfg::kRegsHigh>();
    // with dropout the generator's integer multiplies load the FMA pipe:
    // every exponential goes to the MUFU unit
    constexpr int kPolyPer8 = Cfg::kPolyPer8;
    const int x = (warp >= 8) ? 1 : 0;
    const int quarter = warp & 3;
    const int r_local = quarter * 32 + lane;  // row within the query tile = TMEM lane
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = t_lane + Cfg::col_s(x);
    const uint32_t tO = t_lane + Cfg::col_o(x);
    const uint32_t tP = t_lane + Cfg::col_p(x);
    uint32_t s_cnt = 0, unit_cnt = 0;
    uint32_t q_use = 0;  // units seen: ring index of their Q slot
    uint32_t o_cnt[2] = {0, 0};
    // Staged epilogue: the Q slot whose O store is still reading it.  The
    // storing thread does not wait for that read in place (its warp would lag
    // into the next unit); it waits and releases the slot after its next P,
    // at the next epilogue, or at the end, whichever comes first.
    int pend_slot = -1;
    auto release_pending = [&]() {
      if (Cfg::kEpiTma && r_local == 0 && pend_slot >= 0) {
        bulk_wait_group_read0();
        mbar_arrive(q_empty(pend_slot));
        pend_slot = -1;
      }
    };
    bool ok = true;
    for (int round = 0; ok; ++round) {
      int u = -1;
      ok = fetch_warp(round, u);
      if (!ok || u < 0) break;
      const FwdUnit w = fwd_decode<kPair, kPacked>(p, u);
      const int qs_me = q_use % QSLOTS;
      const uint32_t q_par = (q_use / QSLOTS) & 1;
      ++q_use;
      // this unit's Q is loaded into the pending slot only after its release
      if (pend_slot == qs_me) release_pending();
      if (kPair && x == 1 && !w.has1) {
        // pair with no second tile: nothing to compute or write.  The staged
        // epilogue releases this warpgroup's share of the Q slot, once this
        // unit's Q has landed (so that the arrival counts for this use).
        if constexpr (Cfg::kEpiTma) {
          ok = __all_sync(0xffffffffu, mbar_wait(q_full(qs_me), q_par));
          if (!ok) break;
          if (r_local == 0) mbar_arrive(q_empty(qs_me));
        }
        continue;
      }
      const int i_me = x ? w.i1 : w.i0;           // this warpgroup's query tile
      const int j_end_me = x ? w.j_end1 : w.j_end0;
      const int row = i_me * kTile + r_local;     // query index within the head
      float m_used = -INFINITY;                   // log2 domain, scale folded in
      float l = 0.f;
      int cnt = 0;  // tiles this warpgroup processed
      int k = 0;    // split mode: visit index over both warpgroups
      for (int j = kPair ? 0 : fwd_next(p, w, 0); j < (kPair ? j_end_me : w.j_end);
           j = kPair ? j + 1 : fwd_next(p, w, j + 1), ++k) {
        if (!kPair && (k & 1) != x) continue;
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
        if constexpr (Cfg::kSepP) {
          // S_x is in registers: the issuer may overwrite it with the next S
          tc_fence_before();
          mbar_arrive(s_free(x));
        }
        // element masks on boundary tiles only
        const bool diag = p.causal && (j == i_me);
        const int kv_lim = w.L - j * kTile;  // keys c >= kv_lim are padding
        const bool boundary = diag || kv_lim < kTile;
        // Keys c >= lim are masked.  A 32-key chunk that is masked for every
        // row of the warp (padding past kv_len, or above the diagonal block of
        // the warp's 32 rows) needs no exponentials: bit c of `skip` (the same
        // in all lanes).
        uint32_t skip = 0;
        if (boundary) {
          const int lim = diag ? min(r_local + 1, kv_lim) : kv_lim;
#pragma unroll
          for (int c4 = 0; c4 < kTile / 32; ++c4) {
            if (__all_sync(0xffffffffu, lim <= c4 * 32)) skip |= 1u << c4;
            if (!__all_sync(0xffffffffu, lim >= c4 * 32 + 32)) {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c4 * 32 + e >= lim) sv[c4 * 32 + e] = -INFINITY;
            }
          }
        }
        // row max: eight independent chains of 3-input max, then combined
        float mx8[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) mx8[t] = fmaxf(sv[t], sv[t + 8]);
#pragma unroll
        for (int c = 16; c < kTile; c += 16)
#pragma unroll
          for (int t = 0; t < 8; ++t) mx8[t] = fmax3(mx8[t], sv[c + t], sv[c + 8 + t]);
        const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                               fmaxf(mx8[6], mx8[7]));
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
        const float m_sub = (m_used == -INFINITY) ? 0.f : m_used;
        // P = 2^(s * scale * log2 e - m), two elements per packed FMA.  On
        // interior tiles kPolyPer8 of every 8 pairs use ex2_poly2 on the FMA pipe
        // to offload the MUFU unit; boundary tiles (which hold -inf) use the
        // hardware exp2 throughout.
        const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
        const uint64_t negm2 = f2_pack(-m_sub, -m_sub);
        uint64_t ls4[4] = {0, 0, 0, 0};  // packed partial row sums (0.0f bit pattern)
        auto make_p = [&](auto soft_tag) {
          constexpr bool kSoft = decltype(soft_tag)::value;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t pk[16];
            if constexpr (!kSoft) {  // boundary tiles only: interior ones keep one straight line
              if (skip & (1u << c)) {
                // every key of the chunk is masked for the whole warp: P = 0
#pragma unroll
                for (int e = 0; e < 16; ++e) pk[e] = 0u;
                tmem_st16(tP + c * 16, pk);
                continue;
              }
            }
            [[maybe_unused]] uint4 d4;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              if constexpr (kDrop) {
                // one draw per eight keys: keys c*32 + 8*(e/4) .. +7 of the tile
                // (inline, so that the generator's integer work interleaves with
                // the exponentials)
                if ((e & 3) == 0)
                  d4 = philox4x32_10_rk(static_cast<uint32_t>(j * (kTile / 8) + c * 4 + (e >> 2)),
                                        static_cast<uint32_t>(row), static_cast<uint32_t>(w.bh),
                                        p.drop.offset, p.drop.rk);
              }
              const uint64_t xx =
                  f2_fma(f2_pack(sv[c * 32 + 2 * e], sv[c * 32 + 2 * e + 1]), scale2, negm2);
              float x0, x1, p0, p1;
              f2_unpack(xx, x0, x1);
              if (kSoft && (e & 7) < kPolyPer8) {
                ex2_poly2(x0, x1, p0, p1);
              } else {
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
              }
              ls4[e & 3] = f2_add(ls4[e & 3], f2_pack(p0, p1));
              if constexpr (kDrop) {
                // the row sum above is the softmax's; P V gets the kept P, and
                // the weight w of kept entries is applied with 1 / l at the end
                const uint32_t word = (e & 3) == 0 ? d4.x : (e & 3) == 1 ? d4.y
                                    : (e & 3) == 2 ? d4.z : d4.w;
                p0 = ((word << 16) >= p.drop.t_hi) ? p0 : 0.f;
                p1 = (word >= p.drop.t_hi) ? p1 : 0.f;
              }
              pk[e] = pack_bf16x2(p0, p1);
            }
            tmem_st16(tP + c * 16, pk);
          }
        };
        if constexpr (Cfg::kSepP) {
          // P_x is overwritten below: the previous P V of this warpgroup must
          // have read it (and finished its O update before any rescale of O)
          if (s_cnt >= 2) {
            ok = __all_sync(0xffffffffu, mbar_wait(p_free(x), (s_cnt - 2) & 1));
            if (!ok) break;
          }
          tc_fence_after();
        }
        if (boundary)
          make_p(std::false_type{});
        else
          make_p(std::true_type{});
        {
          const uint64_t s2 = f2_add(f2_add(ls4[0], ls4[1]), f2_add(ls4[2], ls4[3]));
          float s_lo, s_hi;
          f2_unpack(s2, s_lo, s_hi);
          l += s_lo + s_hi;
        }
        // O rescale (rare: the row max grew by more than 2^8) after P is out of
        // registers; it completes before p_full, so before the next P V MMA
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
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full(x));
        release_pending();
        ++cnt;
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) break;
      // rows of a partial last tile beyond N (packed: beyond the sequence) are
      // not output
      const bool row_ok = row < w.nq;
      // O row: [B*H*N][d], or [T][H][d] at column h*d; LSE: [B*H*N], or [H][T]
      uint16_t* const o_row = p.o + (static_cast<long long>(w.tok_base) + row) * p.o_stride +
                              (kPacked ? static_cast<long long>(w.tz) * p.dcols : 0ll);
      float* const lse_ptr = p.lse + (kPacked ? static_cast<long long>(w.tz) * p.T : 0ll) +
                             w.tok_base + row;
      if constexpr (kPair) {
        // ---------------------------------------------------- epilogue (own tile)
        uint4* orow = reinterpret_cast<uint4*>(o_row);
        // Staged: the tile goes through shared memory to one TMA store (the
        // tensor map clips rows beyond N).  A packed tile that crosses its
        // sequence's end is written row by row instead (the rows past the end
        // belong to the next sequence).
        const bool staged = Cfg::kEpiTma && (!kPacked || (i_me + 1) * kTile <= w.nq);
        if (cnt > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(o_full(x), o_cnt[x] & 1));
          ++o_cnt[x];
          if (!ok) break;
          tc_fence_after();
        } else if (Cfg::kEpiTma) {
          // no key tile: the zeros below may be staged over the Q tile only
          // after its load has landed
          ok = __all_sync(0xffffffffu, mbar_wait(q_full(qs_me), q_par));
          if (!ok) break;
        }
        release_pending();
        const float inv_l = (cnt > 0 && l > 0.f) ? (kDrop ? p.drop.w : 1.f) / l : 0.f;
        uint8_t* const stage_row = smem + Cfg::kOffQ +
                                   (qs_me * Cfg::kQPerSlot + x) * Cfg::kTileBytes + r_local * 128;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t pk[16];
          if (cnt > 0) {
            uint32_t r[32];
            tmem_ld32(tO + c * 32, r);
            tmem_wait_ld();
            reg_fence32(r);
#pragma unroll
            for (int e = 0; e < 16; ++e)
              pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                  __uint_as_float(r[2 * e + 1]) * inv_l);
          } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = 0u;
          }
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4) {
            const uint4 val = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
            if (staged) {
              const int g = c * 4 + v4;  // 16-byte granule of the 128-byte row
              *reinterpret_cast<uint4*>(stage_row + ((g ^ (r_local & 7)) << 4)) = val;
            } else if (row_ok && c * 32 + v4 * 8 < p.dcols) {
              orow[c * 4 + v4] = val;
            }
          }
        }
        if (cnt > 0) tc_fence_before();
        if (row_ok)
          *lse_ptr = (cnt > 0 && l > 0.f) ? (m_used + log2f(l)) * kLn2 : -INFINITY;
        if constexpr (Cfg::kEpiTma) {
          if (staged) {
            fence_proxy_async_smem();
            named_bar_sync(8 + x, 128);  // the warpgroup's 128 rows are staged
          }
          if (r_local == 0) {
            if (staged) {
              const int2 yz = tile_yz(kPacked, (kPacked ? w.tok_base : 0) + i_me * kTile, w.tz);
              tma_store_3d(&tm_o, 0, yz.x, yz.y,
                           sbase + Cfg::kOffQ + (qs_me * Cfg::kQPerSlot + x) * Cfg::kTileBytes);
              bulk_commit_group();
              pend_slot = qs_me;  // released once the store has read it
            } else {
              mbar_arrive(q_empty(qs_me));  // the Q slot may be loaded again
            }
          }
        }
      } else {
        // ---------------------------------------------------- merge + epilogue
        // k = visits of the unit: warpgroup 0 processed ceil(k/2), warpgroup 1
        // floor(k/2).  Both warpgroups read both partial outputs: warpgroup x
        // finishes columns [x*D/2, (x+1)*D/2) of every row.
        const int n0 = (k + 1) / 2, n1 = k / 2;
        if (n0 > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(o_full(0), o_cnt[0] & 1));
          ++o_cnt[0];
        }
        if (ok && n1 > 0) {
          ok = __all_sync(0xffffffffu, mbar_wait(o_full(1), o_cnt[1] & 1));
          ++o_cnt[1];
        }
        if (!ok) break;
        tc_fence_after();
        ml_smem[x * kTile + r_local] = make_float2(m_used, cnt > 0 ? l : 0.f);
        mbar_arrive(ml_ready);
        ok = __all_sync(0xffffffffu, mbar_wait(ml_ready, unit_cnt & 1));
        if (!ok) break;
        const float2 ml0 = ml_smem[r_local];
        const float2 ml1 = ml_smem[kTile + r_local];
        const float m = fmaxf(ml0.x, ml1.x);
        const float a0 = (ml0.y > 0.f) ? ex2_approx(ml0.x - m) : 0.f;
        const float a1 = (ml1.y > 0.f) ? ex2_approx(ml1.x - m) : 0.f;
        const float lt = ml0.y * a0 + ml1.y * a1;
        const float inv_l = (lt > 0.f) ? (kDrop ? p.drop.w : 1.f) / lt : 0.f;
        const float f0 = a0 * inv_l, f1 = a1 * inv_l;
        uint4* orow = reinterpret_cast<uint4*>(o_row + x * (D / 2));
        // A warpgroup that processed no tile left its O unwritten: its factor is 0
        // and its values are dropped by a select (never multiplied, in case the
        // unwritten columns hold a NaN pattern).
        const bool use0 = n0 > 0, use1 = n1 > 0;
#pragma unroll 1
        for (int c = 0; c < D / 64; ++c) {
          const uint32_t col = x * (D / 2) + c * 32;
          uint32_t r0[32], r1[32];
          tmem_ld32(t_lane + Cfg::col_o(0) + col, r0);
          tmem_ld32(t_lane + Cfg::col_o(1) + col, r1);
          tmem_wait_ld();
          reg_fence32(r0);
          reg_fence32(r1);
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float a = use0 ? __uint_as_float(r0[2 * e]) * f0 : 0.f;
            const float b = use0 ? __uint_as_float(r0[2 * e + 1]) * f0 : 0.f;
            const float c2 = use1 ? __uint_as_float(r1[2 * e]) * f1 : 0.f;
            const float d2 = use1 ? __uint_as_float(r1[2 * e + 1]) * f1 : 0.f;
            pk[e] = pack_bf16x2(a + c2, b + d2);
          }
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            if (row_ok && static_cast<int>(col) + v4 * 8 < p.dcols)
              orow[c * 4 + v4] =
                  make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
        }
        if (x == 0 && row_ok) *lse_ptr = (lt > 0.f) ? (m + log2f(lt)) * kLn2 : -INFINITY;
        tc_fence_before();
        // neither warpgroup starts the next unit (whose first P V overwrites an O)
        // before both have read both partial outputs
        mbar_arrive(merged);
        ok = __all_sync(0xffffffffu, mbar_wait(merged, unit_cnt & 1));
        ++unit_cnt;
      }
    }
    if (!ok) *abort_flag = 1;
    release_pending();
    if (Cfg::kEpiTma && r_local == 0) bulk_wait_group0();  // O stores complete before exit
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
  if (threadIdx.x == 0) fwd_count_out(p.counter_slot);
}

}  // namespace fa
