// fa_bwd.cuh - backward kernels: recompute the score and probability tiles on
// chip from Q, K, V and the saved log-sum-exp instead of storing them
// ("FlashAttention, Decoded", "The Hardware Picture": recomputation;
// opendecode.dev summary, "The key idea": the matrix is recomputed from the
// tiles in the backward pass).
//
// With S = scale * Q K^T, P = exp(S - LSE), O = P V and upstream gradient dO:
//   dV = P^T dO,  dP = dO V^T,  D_r = sum_x dO_rx O_rx,  dS = P o (dP - D),
//   dQ = scale * dS K,  dK = scale * dS^T Q.
//
// Three launches:
//   fa_bwd_pre_kernel    -D and -LSE*log2(e) per row (per-head padded layout),
//                        zero the f32 dQ accumulator and the work counter
//   fa_bwd_kernel        persistent; a unit is (b, h, 128-key tile j)
//   fa_bwd_dq_kernel     dQ = bf16(scale * accumulator)
//
// fa_bwd_kernel roles (16 warps):
//   warp 0      TMA producer: takes units from a counter shared by all CTAs,
//               decodes each once and publishes it in a shared-memory ring
//               for the other roles; loads K_j, V_j once per unit
//               (double-buffered across units for D = 64) and per visited
//               query tile Q_i with the tile's -LSE2 and -D rows (one ring)
//               and dO_i (a second ring)
//   warp 1      TMEM owner; MMA issuer (one thread).  D = 64: warps 1-3 each
//               issue one share of the MMAs (S^T and dV / dP^T and dK / dQ)
//   warps 4-11  two "dS" warpgroups, one key row per thread (TMEM lane), each
//               on half of the 128 query columns: P^T, dS^T, and the dK (first
//               warpgroup) / dV (second) epilogue of each unit
//   warps 12-15 "dQ" group, one query row per thread: drains dQ partials from
//               TMEM through shared memory into the float32 accumulator in
//               HBM with TMA reduce-adds
// Per visited query tile i, all accumulating in TMEM:
//   S^T  = K_j Q_i^T          (cols   0..127)
//   dP^T = V_j dO_i^T         (cols 128..255)
//   dV  += P^T dO_i           (A = P^T bf16 in TMEM: its own cols 448..511 for
//                             D = 64, over S^T's first 64 cols for D = 128)
//   dK  += dS^T Q_i           (A = dS^T bf16 in TMEM over dP^T's first 64 cols)
//   dQ   = dS K_j             (A = dS from shared memory; result in cols 384..447
//                             for D = 64, over dP^T's cols 128..255 for D = 128)
// dK and dV accumulate in cols 256..256+2D-1 for the whole unit.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

// ---------------------------------------------------------------------------
// preprocess: D_r = sum_x dO_rx O_rx (f32) and LSE_r * log2(e) (+inf for rows
// with no allowed key, so that exp2(s - LSE2) = 0), both stored NEGATED (the
// main kernel adds them), and zero the dQ accumulator.
// ---------------------------------------------------------------------------
// Memory-bound: eight resident blocks per SM (at most 32 registers a thread)
// keep enough loads in flight.
template <int D>
__global__ void __launch_bounds__(256, 8) fa_bwd_pre_kernel(const uint16_t* __restrict__ o,
                                                         const uint16_t* __restrict__ dout,
                                                         const float* __restrict__ lse,
                                                         float* __restrict__ delta,
                                                         float* __restrict__ lse2,
                                                         float4* __restrict__ dq_acc,
                                                         int* __restrict__ work_counter,
                                                         int N, int Np, long long rows_p,
                                                         long long rows, int dcols) {
  pdl_launch_dependents();
  pdl_wait();
  // the main kernel's CTAs take work units from this counter
  if (blockIdx.x == 0 && threadIdx.x == 0) *work_counter = 0;
  constexpr int kLanesPerRow = D / 8;  // one 16-byte chunk (8 bf16) per lane
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const long long warp_global = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;
  const int part = lane % kLanesPerRow;
  // D and LSE2 go to a per-head padded layout (Np = N rounded up to 128 rows
  // per head) so that every 128-row tile of them starts 512-byte aligned;
  // padding rows get -LSE2 = -inf (P = 0) and -D = 0
  for (long long r0 = warp_global * kRowsPerWarp; r0 < rows_p; r0 += nwarps * kRowsPerWarp) {
    const long long pr = r0 + sub;
    long long r = pr;  // when 128 divides N the two layouts coincide
    bool valid = pr < rows_p;
    if (Np != N) {
      const long long bh = pr / Np;
      const int rr = static_cast<int>(pr - bh * Np);
      valid = valid && rr < N;
      r = bh * N + rr;
    }
    float acc = 0.f;
    if (valid && part * 8 < dcols) {  // rows of d = dcols columns (D / 8 lanes cover D)
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + r * dcols) + part);
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + r * dcols) + part);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
        const float2 fb2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (pr < rows_p && part == 0) {
      delta[pr] = valid ? -acc : 0.f;
      const float l = valid ? lse[r] : -INFINITY;
      lse2[pr] = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
    }
  }
  const long long n4 = rows * (dcols / 4);  // the accumulator is [rows][d] float32
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n4;
       e += (long long)gridDim.x * blockDim.x)
    dq_acc[e] = z;
}

// The same for packed variable-length batches: O, dO [T][H][d], LSE [H][T];
// D and LSE2 in the per-head padded layout of the unit grid ([B*H][Np], Np =
// the longest sequence rounded up to 128), rows past a sequence's end as
// padding; the accumulator is [T][H][d] (acc_rows = T * H rows).
template <int D>
__global__ void __launch_bounds__(256, 8) fa_bwd_pre_packed_kernel(
    const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
    const float* __restrict__ lse, float* __restrict__ delta, float* __restrict__ lse2,
    float4* __restrict__ dq_acc, int* __restrict__ work_counter,
    const int32_t* __restrict__ cu_seqlens, int H, int N, int Np, int T, long long rows_p,
    long long acc_rows, int dcols) {
  pdl_launch_dependents();
  pdl_wait();
  if (blockIdx.x == 0 && threadIdx.x == 0) *work_counter = 0;
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const long long warp_global = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kLanesPerRow;
  const int part = lane % kLanesPerRow;
  for (long long r0 = warp_global * kRowsPerWarp; r0 < rows_p; r0 += nwarps * kRowsPerWarp) {
    const long long pr = r0 + sub;
    bool valid = pr < rows_p;
    long long orow = 0, lrow = 0;  // O / dO row (of T * H) and LSE index
    if (valid) {
      const int bh = static_cast<int>(pr / Np);
      const int rr = static_cast<int>(pr - static_cast<long long>(bh) * Np);
      const int b = bh / H, h = bh - b * H;
      const SeqSpan sp = seq_span(cu_seqlens, b, N, T);
      valid = rr < sp.len;
      orow = (static_cast<long long>(sp.start) + rr) * H + h;
      lrow = static_cast<long long>(h) * T + sp.start + rr;
    }
    float acc = 0.f;
    if (valid && part * 8 < dcols) {
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + orow * dcols) + part);
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + orow * dcols) + part);
      const uint32_t av[4] = {a.x, a.y, a.z, a.w};
      const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 fa2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&av[e]));
        const float2 fb2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bv[e]));
        acc = fmaf(fa2.x, fb2.x, acc);
        acc = fmaf(fa2.y, fb2.y, acc);
      }
    }
#pragma unroll
    for (int off = kLanesPerRow / 2; off > 0; off >>= 1)
      acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (pr < rows_p && part == 0) {
      delta[pr] = valid ? -acc : 0.f;
      const float l = valid ? lse[lrow] : -INFINITY;
      lse2[pr] = (l == -INFINITY) ? -INFINITY : -l * kLog2e;
    }
  }
  const long long n4 = acc_rows * (dcols / 4);
  const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n4;
       e += (long long)gridDim.x * blockDim.x)
    dq_acc[e] = z;
}

// dQ = bf16(scale * accumulator), 8 elements per thread per step.
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const float4* __restrict__ dq_acc,
                                                        uint4* __restrict__ dq, float scale,
                                                        long long n8) {
  pdl_launch_dependents();
  pdl_wait();
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n8;
       e += (long long)gridDim.x * blockDim.x) {
    const float4 a = __ldg(dq_acc + 2 * e);
    const float4 b = __ldg(dq_acc + 2 * e + 1);
    dq[e] = make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                       pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
  }
}

// ---------------------------------------------------------------------------
// main backward kernel
// ---------------------------------------------------------------------------
struct BwdParams {
  float* dq_acc;
  const float* delta;  // -D per row
  const float* lse2;   // -LSE * log2(e) per row (-inf: row with no key)
  uint16_t* dk;
  uint16_t* dv;
  const uint8_t* block_mask;
  const int32_t* kv_len;
  uint8_t* visited;
  int B, H, N, n_t;
  int num_units;
  int heads_per_group;  // unit order: see bwd_decode
  // packed variable-length batches (null: the [B][H][N][d] layout), as in
  // FwdParams; o_stride = elements between consecutive rows of one head's
  // dK / dV
  const int32_t* cu_seqlens;
  int T;
  long long o_stride;
  int dcols;  // the tensors' head dimension d (<= D; columns D > d read as zeros)
  int* work_counter;    // next unit to take (zeroed by fa_bwd_pre_kernel)
  int causal;
  float scale;
  float scale_log2;
  DropoutParams drop;   // the forward's mask (kernels instantiated with kDrop)
};

template <int D>
struct BwdCfg {
  static constexpr int kThreads = 512;
  // registers per thread: 128 at launch (512 x 128 = 65536), redistributed:
  //          producer/MMA   two dS warpgroups   dQ warpgroup
  // D = 64:  128 x 104   +  256 x 144        +  128 x 112  = 64512
  // D = 128: 128 x 112   +  256 x 128        +  128 x 144  = 65536
  // (the dQ warpgroup holds a whole float32 dQ row)
  static constexpr uint32_t kRegsLaunch = 128, kRegsLow = (D == 64) ? 104 : 112;
  static constexpr uint32_t kRegsDs = (D == 64) ? 144 : 128;
  static constexpr uint32_t kRegsDq = (D == 64) ? 112 : 144;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kBoxes = D / 64;
  // Q_i (with the tile's -LSE2 and -D rows) and dO_i come through separate
  // rings: dO_i is released after the dV MMA, Q_i after the dK MMA.
  // D = 64: K/V double-buffered across units (the next unit's K and V load
  // while this one runs), two-stage Q and dO rings.  D = 128: one K/V buffer.
  static constexpr bool kSmallD = (D == 64);
  static constexpr int kKvStages = kSmallD ? 2 : 1;
  static constexpr int kQStages = 2;
  static constexpr int kDoStages = kSmallD ? 2 : 1;
  // K/V slot s: K at kOffK + s * kKvSlotBytes, V right after it
  static constexpr int kKvSlotBytes = 2 * kTileBytes;
  static constexpr int kOffK = 0;
  static constexpr int kOffV = kOffK + kTileBytes;
  static constexpr int kOffQ = kOffK + kKvStages * kKvSlotBytes;
  static constexpr int kOffDO = kOffQ + kQStages * kTileBytes;
  // 128 x 128 bf16 dS tile: A operand of the dQ MMA
  static constexpr int kOffDS = kOffDO + kDoStages * kTileBytes;
  // float32 dQ partials staged for the TMA reduce-add: 8 KB per dQ warp
  static constexpr int kOffDQ = kOffDS + kTile * kTile * 2;
  static constexpr int kDqStageBytes = 4 * 8192;
  // per Q stage: -LSE*log2(e) and -D of the stage's 128 query rows
  // D = 64: the dK and dV tiles of a unit are staged here (128-byte swizzled
  // rows, the TMA box layout; 1024-byte aligned like every tile) and written
  // with one TMA store each; D = 128 has no room and stores rows directly
  static constexpr bool kEpiTma = kSmallD;
  static constexpr int kOffEpi = kOffDQ + kDqStageBytes;
  static constexpr int kEpiBytes = kEpiTma ? 2 * kTileBytes : 0;
  static constexpr int kOffRow = kOffEpi + kEpiBytes;
  static constexpr int kRowBytes = kTile * 4;
  // unit records: the producer decodes each work unit once and publishes it
  // here (kUnitRing slots of two int4) for the other roles
  static constexpr int kUnitRing = 4;
  static constexpr int kOffUnit = kOffRow + 2 * kQStages * kRowBytes;
  static constexpr int kOffBar = kOffUnit + kUnitRing * 48;  // records of three int4
  static_assert(kOffEpi % 1024 == 0, "staging tiles must be 1024-byte aligned");
  // kv_full[KVS], kv_empty[KVS], q_full[QS], q_empty[QS], do_full[DS], do_empty[DS],
  // s_full, dp_full, p_full, ds_full, ds_smem_empty, dq_full, dq_empty, dkv_full,
  // drain[3], s_free, p_free, unit_full[UR], unit_empty[UR]
  static constexpr int kNumBars =
      2 * kKvStages + 2 * kQStages + 2 * kDoStages + 13 + 2 * kUnitRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16;
  static_assert(kSmemBytes <= 232448, "shared memory over the per-block limit");
  static constexpr uint32_t kTmemCols = 512;
  // S^T fp32 in cols 0..127; the two math warpgroups each own 64 of them
  // (queries 0..63 and 64..127) and write their P^T (bf16, 32 packed cols)
  // over the start of their own 64: P^T for queries 16k..16k+15 sits at
  // kColS + (k / 4) * 64 + (k % 4) * 8.  The same for dP^T / dS^T at kColDP.
  static constexpr uint32_t kColS = 0;
  static constexpr uint32_t kColDP = 128;
  static constexpr uint32_t kColDK = 256;
  static constexpr uint32_t kColDV = 256 + D;
  // dQ = dS K_j: its own columns when they fit (D = 64), else over dP^T
  // (after the dK MMA has read dS^T there; the next dP^T waits for the drain)
  static constexpr uint32_t kColDQ = (D == 64) ? 384 : 128;
  static constexpr bool kDqAliasesDP = (kColDQ == kColDP);
  // With dQ in its own columns the MMAs split into three independent issue
  // streams (warps 1-3): one issuing thread beside twelve busy math warps is
  // starved of issue slots.  D = 128 (dQ over dP^T) keeps one issuer.
  static constexpr bool kMultiIssue = !kDqAliasesDP;
  // dQ staging: each dQ warp owns 8 KB = two 32 x 32 float32 boxes
  static constexpr int kDqBoxesPerRound = 2;
  static constexpr int kDqRounds = D / 64;
  // TMEM column of the bf16 operand for K-step kk (16 queries) of the dV / dK MMAs
  __device__ static constexpr uint32_t packed_col(uint32_t base, int kk) {
    return base + (kk >> 2) * 64 + (kk & 3) * 8;
  }
  // P^T: D = 64 keeps it in the last 64 columns (32 per warpgroup half), so
  // that the next S^T may be issued once S^T is in the math warps' registers;
  // D = 128 writes it over S^T as described above
  static constexpr uint32_t kColP = kSmallD ? 448 : kColS;
  static constexpr uint32_t kPHalf = kSmallD ? 32 : 64;  // columns between the halves' P^T
  __device__ static constexpr uint32_t p_col(int kk) {
    return kColP + (kk >> 2) * kPHalf + (kk & 3) * 8;
  }
};

struct BwdUnit {
  int bh, b, j, L, i_begin, any, i_first;  // i_first: first visited query tile
  int valid;                                // 0: no unit left (end of the work)
  int tok_base;  // row c of dK / dV is row tok_base + c of the [rows][o_stride] arrays
  int tz;        // TMA third coordinate (the head; packed: h, at column h * d)
  int nq;        // rows of this head (N, or the sequence's length)
  int n_tq;      // query tiles of this head
};

__device__ __forceinline__ bool bwd_tile_on(const BwdParams& p, const BwdUnit& w, int i) {
  if (p.causal && w.j > i) return false;
  if (w.j * kTile >= w.L) return false;
  if (p.block_mask && __ldg(p.block_mask + (size_t)i * p.n_t + w.j) == 0) return false;
  return true;
}

// First visited query tile >= i (or n_tq).
__device__ __forceinline__ int bwd_next(const BwdParams& p, const BwdUnit& w, int i) {
  if (w.j * kTile >= w.L) return w.n_tq;
  for (; i < w.n_tq; ++i)
    if (bwd_tile_on(p, w, i)) return i;
  return w.n_tq;
}

template <bool kPacked = false>
__device__ __forceinline__ BwdUnit bwd_decode(const BwdParams& p, int u) {
  // heads in groups whose Q, dO and dQ accumulator fit in a share of L2; inside
  // a group key tile 0 first (for causal masks it sees the most queries)
  BwdUnit w;
  group_order(u, p.n_t, p.B * p.H, p.heads_per_group, w.bh, w.j);
  w.b = w.bh / p.H;
  int L = p.N;
  if constexpr (kPacked) {
    const SeqSpan sp = seq_span(p.cu_seqlens, w.b, p.N, p.T);
    L = sp.len;
    w.tok_base = sp.start;
    w.tz = w.bh - w.b * p.H;
    w.nq = sp.len;
    w.n_tq = (sp.len + kTile - 1) / kTile;
  } else {
    if (p.kv_len) {
      L = __ldg(p.kv_len + w.b);
      L = L < 0 ? 0 : (L > p.N ? p.N : L);
    }
    w.tok_base = w.bh * p.N;
    w.tz = w.bh;
    w.nq = p.N;
    w.n_tq = p.n_t;
  }
  w.L = L;
  w.i_begin = p.causal ? w.j : 0;
  w.i_first = bwd_next(p, w, w.i_begin);
  w.any = w.i_first < w.n_tq;
  w.valid = 1;
  return w;
}


template <int D, bool kDrop = false, bool kPacked = false>
__global__ void __launch_bounds__(BwdCfg<D>::kThreads, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using Cfg = BwdCfg<D>;
  constexpr int QS = Cfg::kQStages, DOS = Cfg::kDoStages, KVS = Cfg::kKvStages;
  extern __shared__ __align__(1024) uint8_t smem[];
  pdl_launch_dependents();
  if (!smem_aligned_1024(smem)) return;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + Cfg::kOffBar;
  auto kv_full = [&](int s) { return bar0 + 8 * s; };
  auto kv_empty = [&](int s) { return bar0 + 8 * (KVS + s); };
  const uint32_t bar1 = bar0 + 8 * 2 * KVS;
  auto q_full = [&](int s) { return bar1 + 8 * s; };
  auto q_empty = [&](int s) { return bar1 + 8 * (QS + s); };
  auto do_full = [&](int s) { return bar1 + 8 * (2 * QS + s); };
  auto do_empty = [&](int s) { return bar1 + 8 * (2 * QS + DOS + s); };
  const uint32_t s_full = bar1 + 8 * (2 * QS + 2 * DOS);
  const uint32_t dp_full = s_full + 8, p_full = s_full + 16, ds_full = s_full + 24;
  const uint32_t ds_smem_empty = s_full + 32, dq_full = s_full + 40, dq_empty = s_full + 48;
  const uint32_t dkv_full = s_full + 56, drain_bar = s_full + 64;
  auto drain = [&](int r) { return drain_bar + 8 * r; };
  // D = 64: the math groups have S^T in registers (256 arrivals) / dV has read P^T
  const uint32_t s_free = drain_bar + 24, p_free = drain_bar + 32;
  constexpr int UR = Cfg::kUnitRing;
  auto unit_full = [&](int s) { return drain_bar + 40 + 8 * s; };
  auto unit_empty = [&](int s) { return drain_bar + 40 + 8 * (UR + s); };

  static_assert((2 * KVS + 2 * QS + 2 * DOS + 13 + 2 * UR) == Cfg::kNumBars, "barrier layout");
  int4* unit_rec = reinterpret_cast<int4*>(smem + Cfg::kOffUnit);  // [UR][3]
  // the warps that read each unit record: the MMA issuer(s), 8 dS and 4 dQ warps
  constexpr uint32_t kUnitReaders = (Cfg::kMultiIssue ? 3 : 1) + 12;
  auto load_unit = [&](int s) {
    const int4 a = unit_rec[3 * s], b = unit_rec[3 * s + 1];
    BwdUnit w;
    if constexpr (kPacked) {
      const int4 c = unit_rec[3 * s + 2];
      w.tok_base = c.x;
      w.tz = c.y;
      w.nq = c.z;
      w.n_tq = c.w;
    } else {
      w.tok_base = a.x * p.N;
      w.tz = a.x;
      w.nq = p.N;
      w.n_tq = p.n_t;
    }
    w.bh = a.x;
    w.b = a.y;
    w.j = a.z;
    w.L = a.w;
    w.i_begin = b.x;
    w.any = b.y;
    w.i_first = b.z;
    w.valid = b.w;
    return w;
  };
  // one thread's read of round r's unit record (it releases the slot)
  auto fetch_one = [&](int r, BwdUnit& w) -> bool {
    const int s = r % UR;
    if (!mbar_wait(unit_full(s), (r / UR) & 1)) return false;
    w = load_unit(s);
    mbar_arrive(unit_empty(s));
    return true;
  };
  // a whole warp's read (all 32 lanes; lane 0 releases the slot)
  auto fetch_warp = [&](int r, BwdUnit& w) -> bool {
    const int s = r % UR;
    const bool ok = __all_sync(0xffffffffu, mbar_wait(unit_full(s), (r / UR) & 1));
    if (ok) w = load_unit(s);
    __syncwarp();
    if (ok && lane_id() == 0) mbar_arrive(unit_empty(s));
    return ok;
  };
  uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + Cfg::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::kOffMisc + 4);
  auto lse2_smem = [&](int s) {
    return reinterpret_cast<const float4*>(smem + Cfg::kOffRow + s * Cfg::kRowBytes);
  };
  auto delta_smem = [&](int s) {
    return reinterpret_cast<const float4*>(smem + Cfg::kOffRow + (QS + s) * Cfg::kRowBytes);
  };

  const int warp = warp_id();
  const int lane = lane_id();

  if (threadIdx.x == 0) {
    // three issuers: K and V are read by all three, Q and dO by two each
    constexpr uint32_t kIssuers = Cfg::kMultiIssue ? 3 : 1;
    for (int s = 0; s < KVS; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), kIssuers);
    }
    for (int s = 0; s < QS; ++s) {
      mbar_init(q_full(s), 1);
      mbar_init(q_empty(s), Cfg::kMultiIssue ? 2 : 1);
    }
    for (int s = 0; s < DOS; ++s) {
      mbar_init(do_full(s), 1);
      mbar_init(do_empty(s), Cfg::kMultiIssue ? 2 : 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 256);
    mbar_init(ds_full, 256);
    mbar_init(ds_smem_empty, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 128);
    mbar_init(dkv_full, Cfg::kMultiIssue ? 2 : 1);  // dV and dK issuers
    for (int r = 0; r < 3; ++r) mbar_init(drain(r), 1);
    mbar_init(s_free, 256);
    mbar_init(p_free, 1);
    for (int s = 0; s < UR; ++s) {
      mbar_init(unit_full(s), 1);
      mbar_init(unit_empty(s), kUnitReaders);
    }

    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_dq);
    if (Cfg::kEpiTma) {
      prefetch_tmap(&tm_dk);
      prefetch_tmap(&tm_dv);
    }
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
  static_assert(Cfg::kRegsLow * 128 + Cfg::kRegsDs * 256 + Cfg::kRegsDq * 128 <=
                    Cfg::kRegsLaunch * Cfg::kThreads,
                "register split exceeds the launch allocation");

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      uint32_t kv_cnt = 0, q_cnt = 0, do_cnt = 0;
      bool ok = true;
      // Units are taken from a counter shared by all CTAs (reset by the
      // preprocess kernel), in the order bwd_decode gives them (longest
      // first), so that the CTAs finish together whatever the unit lengths.
      // This round's unit and the next one are published (the other roles
      // read a unit's record before its first tile and the next one's at its
      // last); after the work runs out, one record marks the end.
      int published = 0;  // unit records written
      bool ended = false;
      for (int round = 0; ok; ++round) {
        while (!ended && published <= round + 1) {
          const int un = atomicAdd(p.work_counter, 1);
          BwdUnit wr;
          if (un < p.num_units) {
            wr = bwd_decode<kPacked>(p, un);
            // packed batches: key tiles beyond a shorter sequence's end have
            // no rows at all (nothing to compute or write): not published
            if (kPacked && wr.j >= wr.n_tq) continue;
          }
          const int s = published % UR;
          ok = mbar_wait(unit_empty(s), ((published / UR) & 1) ^ 1);
          if (!ok) break;
          if (un < p.num_units) {
            unit_rec[3 * s] = make_int4(wr.bh, wr.b, wr.j, wr.L);
            unit_rec[3 * s + 1] = make_int4(wr.i_begin, wr.any, wr.i_first, 1);
            if constexpr (kPacked) unit_rec[3 * s + 2] = make_int4(wr.tok_base, wr.tz, wr.nq, wr.n_tq);
          } else {
            unit_rec[3 * s + 1] = make_int4(0, 0, 0, 0);
            ended = true;
          }
          mbar_arrive(unit_full(s));
          ++published;
        }
        if (!ok) break;
        const BwdUnit w = load_unit(round % UR);
        if (!w.valid) break;
        if (!w.any) continue;
        const int skv = kv_cnt % KVS;
        ok = mbar_wait(kv_empty(skv), ((kv_cnt / KVS) & 1) ^ 1);
        if (!ok) break;
        ++kv_cnt;
        // TMA rows: packed batches address the sequence's tokens (rows past its
        // end belong to the next sequence: masked keys, queries whose
        // contributions vanish through the padding -LSE2 = -inf)
        const int trow0 = kPacked ? w.tok_base : 0;
        const int2 kyz = tile_yz(kPacked, trow0 + w.j * kTile, w.tz);
        const uint32_t kv_off = skv * Cfg::kKvSlotBytes;
        mbar_arrive_expect_tx(kv_full(skv), 2 * Cfg::kTileBytes);
        for (int bx = 0; bx < Cfg::kBoxes; ++bx) {
          tma_load_3d(sbase + Cfg::kOffK + kv_off + bx * 16384, &tm_k, bx * 64, kyz.x, kyz.y,
                      kv_full(skv));
          tma_load_3d(sbase + Cfg::kOffV + kv_off + bx * 16384, &tm_v, bx * 64, kyz.x, kyz.y,
                      kv_full(skv));
        }
        for (int i = w.i_first; i < w.n_tq && ok; i = bwd_next(p, w, i + 1)) {
          // the tile's -LSE2 and -D rows (per-head padded layout: n_t * 128 rows
          // per head, so the 512-byte block is aligned and stays in the head)
          const long long qrow = (long long)w.bh * p.n_t * kTile + i * kTile;
          const int2 qyz = tile_yz(kPacked, trow0 + i * kTile, w.tz);
          const int sq = q_cnt % QS;
          ok = mbar_wait(q_empty(sq), ((q_cnt / QS) & 1) ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(q_full(sq), Cfg::kTileBytes + 2 * Cfg::kRowBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(sbase + Cfg::kOffQ + sq * Cfg::kTileBytes + bx * 16384, &tm_q, bx * 64,
                        qyz.x, qyz.y, q_full(sq));
          bulk_load(sbase + Cfg::kOffRow + sq * Cfg::kRowBytes, p.lse2 + qrow, Cfg::kRowBytes,
                    q_full(sq));
          bulk_load(sbase + Cfg::kOffRow + (QS + sq) * Cfg::kRowBytes, p.delta + qrow,
                    Cfg::kRowBytes, q_full(sq));
          ++q_cnt;
          const int so = do_cnt % DOS;
          ok = mbar_wait(do_empty(so), ((do_cnt / DOS) & 1) ^ 1);
          if (!ok) break;
          mbar_arrive_expect_tx(do_full(so), Cfg::kTileBytes);
          for (int bx = 0; bx < Cfg::kBoxes; ++bx)
            tma_load_3d(sbase + Cfg::kOffDO + so * Cfg::kTileBytes + bx * 16384, &tm_do, bx * 64,
                        qyz.x, qyz.y, do_full(so));
          ++do_cnt;
        }
        if (*abort_flag) ok = false;
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 1 && !Cfg::kMultiIssue) {
    // ------------------------------------------------- MMA issuer (D = 128)
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      constexpr uint32_t idesc_kk = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idesc_tn = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A in TMEM)
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 1, 1);    // dQ (both MN-major)
      uint32_t kv_cnt = 0, q_cnt = 0, do_cnt = 0, p_cnt = 0, ds_cnt = 0;
      uint32_t dq_cnt = 0, dq_drained = 0;  // dQ MMAs issued / drained by the dQ group
      bool ok = true;
      // one descriptor base per operand; offsets are added to the start-address field
      const uint64_t dk_k = sw128_desc(sbase + Cfg::kOffK, 16, 1024);     // K_j, K-major
      const uint64_t dv_k = sw128_desc(sbase + Cfg::kOffV, 16, 1024);     // V_j, K-major
      const uint64_t dq_k0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);    // Q_i, K-major
      const uint64_t ddo_k0 = sw128_desc(sbase + Cfg::kOffDO, 16, 1024);  // dO_i, K-major
      const uint64_t dq_m0 = sw128_desc(sbase + Cfg::kOffQ, 16384, 1024);    // Q_i, MN-major
      const uint64_t ddo_m0 = sw128_desc(sbase + Cfg::kOffDO, 16384, 1024);  // dO_i, MN-major
      const uint64_t dk_m = sw128_desc(sbase + Cfg::kOffK, 16384, 1024);     // K_j, MN-major
      const uint64_t dds_m = sw128_desc(sbase + Cfg::kOffDS, 16384, 1024);   // dS, MN-major
      // waits until every issued dQ has been read out of TMEM by the dQ group
      auto drain_dq = [&]() -> bool {
        while (dq_drained < dq_cnt) {
          if (!mbar_wait(dq_empty, dq_drained & 1)) return false;
          ++dq_drained;
        }
        return true;
      };
      // S^T = K_j Q_i^T for the Q tile in ring slot c
      auto issue_st = [&](uint32_t c, const BwdUnit& w, int i) -> bool {
        const int sq = c % QS;
        if (!mbar_wait(q_full(sq), (c / QS) & 1)) return false;
        tc_fence_after();
        const uint32_t q_off = (sq * Cfg::kTileBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::kColS, dk_k + off, dq_k0 + q_off + off, idesc_kk, kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        if (p.visited) p.visited[((size_t)w.bh * p.n_t + i) * p.n_t + w.j] = 1;
        return true;
      };
      // dP^T = V_j dO_i^T for the dO tile in ring slot c
      auto issue_dpt = [&](uint32_t c) -> bool {
        const int so = c % DOS;
        if (!mbar_wait(do_full(so), (c / DOS) & 1)) return false;
        if (Cfg::kDqAliasesDP && !drain_dq()) return false;  // dP^T overwrites the last dQ
        tc_fence_after();
        const uint32_t do_off = (so * Cfg::kTileBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::kColDP, dv_k + off, ddo_k0 + do_off + off, idesc_kk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(dp_full);
        return true;
      };
      for (int round = 0; ok; ++round) {
        BwdUnit w;
        ok = fetch_one(round, w);
        if (!ok || !w.valid) break;
        if (!w.any) continue;
        ok = mbar_wait(kv_full(0), kv_cnt & 1);
        ++kv_cnt;
        if (!ok) break;
        // Per query tile t the issue order is
        //   dV(t) S^T(t+1) | dK(t) dQ(t) dP^T(t+1)
        // S^T's columns are free once the dV MMA has read P^T(t) from them (the
        // math warps keep their own copy of P in registers for dS), so S^T(t+1)
        // is computed while the math warps work on dS(t), and their P phase of
        // tile t+1 overlaps the dK / dQ MMAs of tile t; dP^T(t+1) follows dK(t),
        // which reads dS^T(t) from the dP^T columns, and the dQ drain.
        int i = w.i_first;
        ok = issue_st(q_cnt, w, i) && issue_dpt(do_cnt);
        for (int t = 0; ok && i < w.n_tq; ++t) {
          const int inext = bwd_next(p, w, i + 1);
          const int sq = q_cnt % QS, so = do_cnt % DOS;
          const uint32_t q_off = (sq * Cfg::kTileBytes) >> 4;
          const uint32_t do_off = (so * Cfg::kTileBytes) >> 4;
          // dV += P^T dO_i
          ok = mbar_wait(p_full, p_cnt & 1);
          ++p_cnt;
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + Cfg::kColDV, tmem + Cfg::p_col(kk),
                    ddo_m0 + do_off + ((kk * 2048) >> 4), idesc_tn,
                    (t > 0 || kk > 0) ? 1u : 0u);
          umma_commit(do_empty(so));
          ++do_cnt;
          if (inext < w.n_tq) {
            ok = issue_st(q_cnt + 1, w, inext);
            if (!ok) break;
          }
          ok = mbar_wait(ds_full, ds_cnt & 1);
          ++ds_cnt;
          if (!ok) break;
          tc_fence_after();
          // dK += dS^T Q_i
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ts(tmem + Cfg::kColDK, tmem + Cfg::packed_col(Cfg::kColDP, kk),
                    dq_m0 + q_off + ((kk * 2048) >> 4), idesc_tn,
                    (t > 0 || kk > 0) ? 1u : 0u);
          umma_commit(q_empty(sq));
          ++q_cnt;
          // dQ = dS K_j
          if (!Cfg::kDqAliasesDP && !drain_dq()) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            umma_ss(tmem + Cfg::kColDQ, dds_m + ((kk * 2048) >> 4), dk_m + ((kk * 2048) >> 4),
                    idesc_dq, kk > 0 ? 1u : 0u);
          umma_commit(dq_full);
          umma_commit(ds_smem_empty);
          ++dq_cnt;
          if (inext < w.n_tq) {
            ok = issue_dpt(do_cnt);
            if (!ok) break;
          }
          i = inext;
          if (*abort_flag) ok = false;
        }
        if (!ok) break;
        umma_commit(kv_empty(0));
        umma_commit(dkv_full);
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain_bar);
      mbar_wait(drain_bar, 0);
    }
    __syncwarp();
  } else if (Cfg::kMultiIssue && warp <= 3) {
    // ------------------------------- MMA issuers, three warps (D = 64)
    // role 0: S^T and dV; role 1: dP^T and dK; role 2: dQ.  Each role keeps
    // the read-before-overwrite order of its own TMEM columns in its issue
    // order; what it needs from the other roles comes through the math
    // groups' barriers.  S^T(t+1) follows the math groups' read of S^T(t)
    // (s_free) and dP^T(t+1) follows dK(t), also across the boundary to the
    // next unit, whose K and V are already loaded in the other K/V slot.
    setmaxnreg_dec<Cfg::kRegsLow>();
    if (lane == 0) {
      const int role = warp - 1;
      constexpr uint32_t idesc_kk = idesc_bf16_f32(128, 128, 0, 0);  // S^T, dP^T
      constexpr uint32_t idesc_tn = idesc_bf16_f32(128, D, 0, 1);    // dV, dK (A in TMEM)
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, 1, 1);    // dQ (both MN-major)
      const uint64_t dk_k0 = sw128_desc(sbase + Cfg::kOffK, 16, 1024);    // K_j, K-major
      const uint64_t dv_k0 = sw128_desc(sbase + Cfg::kOffV, 16, 1024);    // V_j, K-major
      const uint64_t dq_k0 = sw128_desc(sbase + Cfg::kOffQ, 16, 1024);    // Q_i, K-major
      const uint64_t ddo_k0 = sw128_desc(sbase + Cfg::kOffDO, 16, 1024);  // dO_i, K-major
      const uint64_t dq_m0 = sw128_desc(sbase + Cfg::kOffQ, 16384, 1024);    // Q_i, MN-major
      const uint64_t ddo_m0 = sw128_desc(sbase + Cfg::kOffDO, 16384, 1024);  // dO_i, MN-major
      const uint64_t dk_m0 = sw128_desc(sbase + Cfg::kOffK, 16384, 1024);    // K_j, MN-major
      const uint64_t dds_m = sw128_desc(sbase + Cfg::kOffDS, 16384, 1024);   // dS, MN-major
      uint32_t kv_cnt = 0, q_cnt = 0, do_cnt = 0, t_cnt = 0;  // t_cnt: tiles (barrier phases)
      bool ok = true;
      // role 0: S^T = K Q_i^T, K from K/V slot skv, Q of ring index c
      auto issue_st = [&](uint32_t c, int skv, const BwdUnit& w, int i) -> bool {
        const int sq = c % QS;
        if (!mbar_wait(q_full(sq), (c / QS) & 1)) return false;
        tc_fence_after();
        const uint32_t q_off = (sq * Cfg::kTileBytes) >> 4;
        const uint32_t k_off = (skv * Cfg::kKvSlotBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::kColS, dk_k0 + k_off + off, dq_k0 + q_off + off, idesc_kk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(s_full);
        umma_commit(q_empty(sq));  // this role's use of Q_i
        if (p.visited) p.visited[((size_t)w.bh * p.n_t + i) * p.n_t + w.j] = 1;
        return true;
      };
      // role 1: dP^T = V dO_i^T, V from K/V slot skv, dO of ring index c
      auto issue_dpt = [&](uint32_t c, int skv) -> bool {
        const int so = c % DOS;
        if (!mbar_wait(do_full(so), (c / DOS) & 1)) return false;
        tc_fence_after();
        const uint32_t do_off = (so * Cfg::kTileBytes) >> 4;
        const uint32_t v_off = (skv * Cfg::kKvSlotBytes) >> 4;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * 16384 + (kk & 3) * 32) >> 4;
          umma_ss(tmem + Cfg::kColDP, dv_k0 + v_off + off, ddo_k0 + do_off + off, idesc_kk,
                  kk > 0 ? 1u : 0u);
        }
        umma_commit(dp_full);
        umma_commit(do_empty(so));  // this role's use of dO_i
        return true;
      };
      bool pre = false;  // roles 0 / 1: this unit's first S^T / dP^T already issued
      bool have_next = false;  // the next round's record was read at the look-ahead
      BwdUnit w_next;
      for (int round = 0; ok; ++round) {
        BwdUnit w;
        if (have_next) {
          w = w_next;
          have_next = false;
        } else {
          ok = fetch_one(round, w);
          if (!ok) break;
        }
        if (!w.valid) break;
        if (!w.any) continue;
        const int skv = kv_cnt % KVS;
        if (!pre) ok = mbar_wait(kv_full(skv), (kv_cnt / KVS) & 1);
        ++kv_cnt;
        if (!ok) break;
        const uint32_t k_off = (skv * Cfg::kKvSlotBytes) >> 4;
        int i = w.i_first;
        if (!pre) {
          if (role == 0) ok = issue_st(q_cnt, skv, w, i);
          if (role == 1) ok = issue_dpt(do_cnt, skv);
          if (!ok) break;
        }
        bool pre_next = false;
        // the first tile of the next unit, for the look-ahead at the last tile
        auto next_unit_first = [&](BwdUnit& wn, int& in) -> bool {
          if (!fetch_one(round + 1, w_next)) {
            ok = false;
            return false;
          }
          have_next = true;
          wn = w_next;
          if (!wn.valid || !wn.any) return false;
          in = wn.i_first;
          if (!mbar_wait(kv_full(kv_cnt % KVS), (kv_cnt / KVS) & 1)) {
            ok = false;
            return false;
          }
          return true;
        };
        for (int t = 0; ok && i < w.n_tq; ++t) {
          const int inext = bwd_next(p, w, i + 1);
          const int sq = q_cnt % QS, so = do_cnt % DOS;
          if (role == 0) {
            // S^T(t+1) once the math groups hold S^T(t) in registers
            ok = mbar_wait(s_free, t_cnt & 1);
            if (!ok) break;
            if (inext < w.n_tq) {
              ok = issue_st(q_cnt + 1, skv, w, inext);
            } else {
              BwdUnit wn;
              int in;
              if (next_unit_first(wn, in)) {
                ok = issue_st(q_cnt + 1, kv_cnt % KVS, wn, in);
                pre_next = true;
              }
            }
            if (!ok) break;
            // dV += P^T dO_i once P^T is in TMEM (dO_i awaited here as well:
            // the roles run independently)
            ok = mbar_wait(p_full, t_cnt & 1) && mbar_wait(do_full(so), (do_cnt / DOS) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t do_off = (so * Cfg::kTileBytes) >> 4;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              umma_ts(tmem + Cfg::kColDV, tmem + Cfg::p_col(kk),
                      ddo_m0 + do_off + ((kk * 2048) >> 4), idesc_tn,
                      (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(p_free);
            umma_commit(do_empty(so));
          } else if (role == 1) {
            // dK += dS^T Q_i, then dP^T(t+1) over dS^T(t) (issue order)
            ok = mbar_wait(ds_full, t_cnt & 1) && mbar_wait(q_full(sq), (q_cnt / QS) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t q_off = (sq * Cfg::kTileBytes) >> 4;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              umma_ts(tmem + Cfg::kColDK, tmem + Cfg::packed_col(Cfg::kColDP, kk),
                      dq_m0 + q_off + ((kk * 2048) >> 4), idesc_tn,
                      (t > 0 || kk > 0) ? 1u : 0u);
            umma_commit(q_empty(sq));
            if (inext < w.n_tq) {
              ok = issue_dpt(do_cnt + 1, skv);
            } else {
              umma_commit(dkv_full);  // dK of the unit complete (with role 0's dV)
              BwdUnit wn;
              int in;
              if (next_unit_first(wn, in)) {
                ok = issue_dpt(do_cnt + 1, kv_cnt % KVS);
                pre_next = true;
              }
            }
            if (!ok) break;
          } else {
            // dQ = dS K once dS is in shared memory and the previous dQ has
            // been drained from its columns
            ok = mbar_wait(ds_full, t_cnt & 1);
            if (ok && t_cnt > 0) ok = mbar_wait(dq_empty, (t_cnt - 1) & 1);
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              umma_ss(tmem + Cfg::kColDQ, dds_m + ((kk * 2048) >> 4),
                      dk_m0 + k_off + ((kk * 2048) >> 4), idesc_dq, kk > 0 ? 1u : 0u);
            umma_commit(dq_full);
            umma_commit(ds_smem_empty);
          }
          ++t_cnt;
          ++q_cnt;
          ++do_cnt;
          i = inext;
          if (*abort_flag) ok = false;
        }
        if (!ok) break;
        if (role == 0) umma_commit(dkv_full);  // dV of the unit complete
        umma_commit(kv_empty(skv));            // this role's use of the unit's K/V
        pre = pre_next;
      }
      if (!ok) *abort_flag = 1;
      umma_commit(drain(role));
      mbar_wait(drain(role), 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    setmaxnreg_dec<Cfg::kRegsLow>();  // idle warps of the first warpgroup
  } else if (warp < 12) {
    // ------------------------------------------------------------ dS groups
    // Warpgroup h (warps 4-7: h = 0, warps 8-11: h = 1) handles queries
    // 64h..64h+63 of every key row; one key row per thread (TMEM lane).
    if constexpr (Cfg::kRegsDs > Cfg::kRegsLaunch) setmaxnreg_inc<Cfg::kRegsDs>();
    // every exponential of the backward pass goes to the MUFU unit: moving a
    // quarter of them to the FMA pipe (ex2_poly2, as the forward pass does)
    // was 3% slower at D = 64 and no faster at D = 128
    const int h = (warp >= 8) ? 1 : 0;
    const int quarter = warp & 3;
    const int kr = quarter * 32 + lane;  // key row within the tile
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t tS = t_lane + Cfg::kColS + h * 64;    // this half's S^T columns
    const uint32_t tP = t_lane + Cfg::kColP + h * Cfg::kPHalf;  // this half's P^T (bf16)
    const uint32_t tDP = t_lane + Cfg::kColDP + h * 64;  // this half's dP^T / dS^T columns
    uint8_t* ds_rowp = smem + Cfg::kOffDS + h * 16384 + kr * 128;
    uint32_t s_cnt = 0, dp_cnt = 0, dsm_cnt = 0, dkv_cnt = 0, q_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      BwdUnit w;
      ok = fetch_warp(round, w);
      if (!ok || !w.valid) break;
      const int c_key = w.j * kTile + kr;  // key index within the head
      const long long krow = static_cast<long long>(w.tok_base) + c_key;
      const int hcol = kPacked ? w.tz : 0;
      // warpgroup 0 writes the dK row, warpgroup 1 the dV row
      uint4* out_row = reinterpret_cast<uint4*>((h ? p.dv : p.dk) + krow * p.o_stride +
                                                static_cast<long long>(hcol) * p.dcols);
      // key rows of a partial last tile beyond N (packed: beyond the sequence)
      // belong to no output
      const bool key_row_ok = c_key < w.nq;
      // The TMA store writes all 128 rows of the tile; the 3-D tensor map
      // clips them at N, but in a packed batch rows past the sequence's end
      // belong to the next sequence: such a tile is written row by row.
      const bool epi_tma = Cfg::kEpiTma && !(kPacked && (w.j + 1) * kTile > w.nq);
      if (!w.any) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c)
          if (key_row_ok && c * 8 < p.dcols) out_row[c] = make_uint4(0, 0, 0, 0);
        continue;
      }
      const bool key_valid = c_key < w.L;
      for (int i = w.i_first; i < w.n_tq; i = bwd_next(p, w, i + 1)) {
        const int sq = q_cnt % QS;
        ++q_cnt;
        const float4* lz4 = lse2_smem(sq) + h * 16;   // -LSE2
        const float4* dz4 = delta_smem(sq) + h * 16;  // -D
        const bool diag = p.causal && (i == w.j);
        // A partial last query tile needs no mask: a query beyond N has Q and dO
        // rows read as zero (so S = dP = 0) and padding entries -LSE2 = -inf,
        // -D = 0, so P is 0 (or, on the polynomial path, clamped to about
        // 2^-126) and dS = P * 0 = 0; its contributions P dO, dS Q and dS K are
        // exactly zero and nothing in them can be infinite or NaN.
        // dropout: this key's keep bits for the half's 64 queries (bit q of kb[c]
        // is query i*128 + h*64 + c*32 + q), drawn while the S^T MMA runs.  A
        // draw covers eight keys of one query, so the eight lanes of a key group
        // share the work: lane slot s draws queries s + 8t (t < 4) and packs the
        // keep bits into R (bit 8t + k = key k of the group, query s + 8t); each
        // lane then reads R from the group's eight lanes and keeps its own key's
        // bits.  All 32 lanes take part: this sits outside the per-lane branches.
        uint32_t kb[2] = {0u, 0u};
        if constexpr (kDrop) {
          const int slot = lane & 7;
          const int src0 = lane & ~7;
          const int kk = kr & 7;  // this lane's key within its group of eight
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t R = 0;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint4 d4 = philox4x32_10_rk(
                  static_cast<uint32_t>(c_key >> 3),
                  static_cast<uint32_t>(i * kTile + h * 64 + c * 32 + slot + 8 * t),
                  static_cast<uint32_t>(w.bh), p.drop.offset, p.drop.rk);
              R |= keep_bits8(d4, p.drop.t_hi) << (8 * t);
            }
            uint32_t bits = 0;
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
              const uint32_t Rs = __shfl_sync(0xffffffffu, R, src0 | s8);
              bits |= ((Rs >> kk) & 0x01010101u) << s8;  // queries s8 + 8t
            }
            kb[c] = bits;
          }
        }
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, s_cnt & 1));
        ++s_cnt;
        if (!ok) break;
        tc_fence_after();
        // P^T: p[q] = exp2(S^T[kr][q] * scale*log2e - LSE2[q]); masked -> 0.
        // Three kinds of row: a key beyond kv_len (all zero, no exponentials),
        // the causal diagonal tile (element mask), and the rest (no mask).
        // P (packed bf16) stays in registers for the dS phase (with dropout the
        // undropped P; TMEM gets the kept P^T for the dV MMA), so the dS phase
        // does not read P^T back and, at D = 128, the next S^T may be written over
        // P^T as soon as the dV MMA has read it
        uint32_t pu[2][16];
        {
          uint32_t r[2][32];
          tmem_ld32(tS, r[0]);
          tmem_ld32(tS + 32, r[1]);
          tmem_wait_ld();
          reg_fence32(r[0]);
          reg_fence32(r[1]);
          bool wait_ok = true;
          if constexpr (Cfg::kSmallD) {
            // S^T is in registers: the next S^T may be issued over it.  P^T is
            // written below: the previous dV must have read it.
            tc_fence_before();
            mbar_arrive(s_free);
            if (s_cnt >= 2) wait_ok = mbar_wait(p_free, (s_cnt - 2) & 1);
            tc_fence_after();
          }
          ok = __all_sync(0xffffffffu, wait_ok);
          const uint64_t scale2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t pk[16];
            // kind: 0 = no mask, 1 = causal diagonal tile (element mask)
            auto make_p = [&](auto kind_tag) {
              constexpr int kKind = decltype(kind_tag)::value;
#pragma unroll
              for (int e4 = 0; e4 < 8; ++e4) {
                const float4 nl = lz4[c * 8 + e4];  // -LSE2 of 4 queries
                const uint64_t xa = f2_fma(
                    f2_pack(__uint_as_float(r[c][4 * e4]), __uint_as_float(r[c][4 * e4 + 1])),
                    scale2, f2_pack(nl.x, nl.y));
                const uint64_t xb = f2_fma(
                    f2_pack(__uint_as_float(r[c][4 * e4 + 2]), __uint_as_float(r[c][4 * e4 + 3])),
                    scale2, f2_pack(nl.z, nl.w));
                float x0, x1, x2, x3, p0, p1, p2, p3;
                f2_unpack(xa, x0, x1);
                f2_unpack(xb, x2, x3);
                p0 = ex2_approx(x0);
                p1 = ex2_approx(x1);
                p2 = ex2_approx(x2);
                p3 = ex2_approx(x3);
                if (kKind == 1) {
                  const int q0 = h * 64 + c * 32 + 4 * e4;  // query within the tile
                  p0 = (kr > q0) ? 0.f : p0;
                  p1 = (kr > q0 + 1) ? 0.f : p1;
                  p2 = (kr > q0 + 2) ? 0.f : p2;
                  p3 = (kr > q0 + 3) ? 0.f : p3;
                }
                // dS gets the whole P; with dropout, dV the kept P (w is applied in
                // its epilogue)
                pu[c][2 * e4] = pack_bf16x2(p0, p1);
                pu[c][2 * e4 + 1] = pack_bf16x2(p2, p3);
                if constexpr (kDrop) {
                  const uint32_t b4 = kb[c] >> (4 * e4);
                  p0 = (b4 & 1u) ? p0 : 0.f;
                  p1 = (b4 & 2u) ? p1 : 0.f;
                  p2 = (b4 & 4u) ? p2 : 0.f;
                  p3 = (b4 & 8u) ? p3 : 0.f;
                  pk[2 * e4] = pack_bf16x2(p0, p1);
                  pk[2 * e4 + 1] = pack_bf16x2(p2, p3);
                } else {
                  pk[2 * e4] = pu[c][2 * e4];
                  pk[2 * e4 + 1] = pu[c][2 * e4 + 1];
                }
              }
            };
            // no allowed entry: a padding key, or (diagonal tile) a query chunk
            // that lies wholly before the warp's 32 keys
            if (!key_valid || (diag && quarter > 2 * h + c)) {
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                pk[e] = 0u;
                pu[c][e] = 0u;
              }
            } else if (diag) {
              make_p(std::integral_constant<int, 1>{});
            } else {
              make_p(std::integral_constant<int, 0>{});
            }
            __syncwarp();
            tmem_st16(tP + c * 16, pk);
          }
        }
        if (!ok) break;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(p_full);
        // dS^T: ds[q] = p[q] * (dP^T[kr][q] - D[q]), p read back (bf16) from TMEM
        // (rows beyond kv_len have p = 0, hence ds = 0)
        ok = __all_sync(0xffffffffu, mbar_wait(dp_full, dp_cnt & 1));
        ++dp_cnt;
        if (!ok) break;
        ok = __all_sync(0xffffffffu, mbar_wait(ds_smem_empty, (dsm_cnt & 1) ^ 1));
        ++dsm_cnt;
        if (!ok) break;
        tc_fence_after();
        {
          // dropout: one 32-query chunk of dP^T at a time (fewer registers live
          // next to the keep bits); otherwise both chunks at once
          uint32_t r[2][32];
          if constexpr (kDrop) {
            tmem_ld32(tDP, r[0]);
          } else {
            tmem_ld32(tDP, r[0]);
            tmem_ld32(tDP + 32, r[1]);
            tmem_wait_ld();
            reg_fence32(r[0]);
            reg_fence32(r[1]);
          }
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            if constexpr (kDrop) {
              if (c == 1) tmem_ld32(tDP + 32, r[1]);
              tmem_wait_ld();
              reg_fence32(r[c]);
            }
            uint32_t pk[16];
#pragma unroll
            for (int e4 = 0; e4 < 8; ++e4) {
              const float4 nd = dz4[c * 8 + e4];  // -D of 4 queries
              uint64_t ta, tb;
              uint32_t pa, pb;
              if constexpr (kDrop) {
                // dropout: the gradient reaching P is dP * Z * w
                const uint32_t b4 = kb[c] >> (4 * e4);
                const float z0 = (b4 & 1u) ? p.drop.w : 0.f, z1 = (b4 & 2u) ? p.drop.w : 0.f;
                const float z2 = (b4 & 4u) ? p.drop.w : 0.f, z3 = (b4 & 8u) ? p.drop.w : 0.f;
                ta = f2_fma(
                    f2_pack(__uint_as_float(r[c][4 * e4]), __uint_as_float(r[c][4 * e4 + 1])),
                    f2_pack(z0, z1), f2_pack(nd.x, nd.y));
                tb = f2_fma(
                    f2_pack(__uint_as_float(r[c][4 * e4 + 2]), __uint_as_float(r[c][4 * e4 + 3])),
                    f2_pack(z2, z3), f2_pack(nd.z, nd.w));
                pa = pu[c][2 * e4];  // the undropped P
                pb = pu[c][2 * e4 + 1];
              } else {
                ta = f2_add(
                    f2_pack(__uint_as_float(r[c][4 * e4]), __uint_as_float(r[c][4 * e4 + 1])),
                    f2_pack(nd.x, nd.y));
                tb = f2_add(
                    f2_pack(__uint_as_float(r[c][4 * e4 + 2]), __uint_as_float(r[c][4 * e4 + 3])),
                    f2_pack(nd.z, nd.w));
                pa = pu[c][2 * e4];
                pb = pu[c][2 * e4 + 1];
              }
              float d0, d1, d2, d3;
              f2_unpack(f2_mul(ta, bf16x2_to_f2(pa)), d0, d1);
              f2_unpack(f2_mul(tb, bf16x2_to_f2(pb)), d2, d3);
              pk[2 * e4] = pack_bf16x2(d0, d1);
              pk[2 * e4 + 1] = pack_bf16x2(d2, d3);
            }
            tmem_st16(tDP + c * 16, pk);
            // shared-memory copy for the dQ MMA: [key][query], this half's 64-query
            // chunk, 128-byte rows, 16-byte granules swizzled by (key & 7)
#pragma unroll
            for (int g4 = 0; g4 < 4; ++g4) {
              const int g = c * 4 + g4;
              *reinterpret_cast<uint4*>(ds_rowp + ((g ^ (kr & 7)) << 4)) =
                  make_uint4(pk[4 * g4], pk[4 * g4 + 1], pk[4 * g4 + 2], pk[4 * g4 + 3]);
            }
          }
        }
        fence_proxy_async_smem();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(ds_full);
        if (*abort_flag) { ok = false; break; }
      }
      if (!ok) break;
      // ---------------------------------------------- dK (h = 0) / dV (h = 1) epilogue
      ok = __all_sync(0xffffffffu, mbar_wait(dkv_full, dkv_cnt & 1));
      ++dkv_cnt;
      if (!ok) break;
      tc_fence_after();
      if (epi_tma) {
        // this warp's previous TMA store (issued by its first lane, not awaited
        // then) has read the warp's 32 staged rows
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
      }
      const float mul = h ? (kDrop ? p.drop.w : 1.f) : p.scale;  // dV: dropout weight
      const uint32_t tAcc = t_lane + (h ? Cfg::kColDV : Cfg::kColDK);
      uint8_t* epi_row = smem + Cfg::kOffEpi + h * Cfg::kTileBytes + kr * 128;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tAcc + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * mul, __uint_as_float(r[2 * e + 1]) * mul);
#pragma unroll
        for (int v4 = 0; v4 < 4; ++v4) {
          const uint4 val = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
          if (epi_tma) {
            const int g = c * 4 + v4;  // 16-byte granule of the 128-byte row
            *reinterpret_cast<uint4*>(epi_row + ((g ^ (kr & 7)) << 4)) = val;
          } else if (key_row_ok && c * 32 + v4 * 8 < p.dcols) {
            out_row[c * 4 + v4] = val;
          }
        }
      }
      tc_fence_before();
      if (epi_tma) {
        // the warp's 32 rows are staged: its first lane stores them as one
        // 32-row box (the next epilogue waits for the store's read of them),
        // so no warp waits for another
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int2 yz =
              tile_yz(kPacked, (kPacked ? w.tok_base : 0) + w.j * kTile + quarter * 32, w.tz);
          tma_store_3d(h ? &tm_dv : &tm_dk, 0, yz.x, yz.y,
                       smem_u32(smem + Cfg::kOffEpi + h * Cfg::kTileBytes + quarter * 4096));
          bulk_commit_group();
        }
      }
    }
    if (!ok) *abort_flag = 1;
    if (Cfg::kEpiTma && lane == 0) bulk_wait_group0();  // stores complete before exit
  } else {
    // ------------------------------------------------------------ dQ group
    // Drains dQ partials: TMEM -> registers -> its own shared-memory staging
    // area -> TMA reduce-add into the float32 accumulator, in 32 x 32 boxes
    // (128-byte swizzled rows).
    if constexpr (Cfg::kRegsDq > Cfg::kRegsLaunch)
      setmaxnreg_inc<Cfg::kRegsDq>();
    else if constexpr (Cfg::kRegsDq < Cfg::kRegsLaunch)
      setmaxnreg_dec<Cfg::kRegsDq>();
    const int quarter = warp & 3;  // rows quarter*32 .. +31 of the query tile
    const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
    uint8_t* stage = smem + Cfg::kOffDQ + quarter * (Cfg::kDqBoxesPerRound * 4096);
    const uint32_t stage_u32 = smem_u32(stage);
    uint32_t dq_cnt = 0;
    bool ok = true;
    for (int round = 0; ok; ++round) {
      BwdUnit w;
      ok = fetch_warp(round, w);
      if (!ok || !w.valid) break;
      if (!w.any) continue;
      for (int i = w.i_first; i < w.n_tq; i = bwd_next(p, w, i + 1)) {
        ok = __all_sync(0xffffffffu, mbar_wait(dq_full, dq_cnt & 1));
        ++dq_cnt;
        if (!ok) break;
        tc_fence_after();
        uint32_t r[D / 32][32];
#pragma unroll
        for (int c = 0; c < D / 32; ++c) tmem_ld32(t_lane + Cfg::kColDQ + c * 32, r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) reg_fence32(r[c]);
        tc_fence_before();
        mbar_arrive(dq_empty);
        // row of the accumulator's tensor map (packed: token row; rows past the
        // sequence's end receive exact or ~1e-38-scaled zeros, see above)
        const int2 yz = tile_yz(kPacked, (kPacked ? w.tok_base : 0) + i * kTile + quarter * 32, w.tz);
#pragma unroll
        for (int rd = 0; rd < Cfg::kDqRounds; ++rd) {
#pragma unroll
          for (int bxi = 0; bxi < Cfg::kDqBoxesPerRound; ++bxi) {
            const int c = rd * Cfg::kDqBoxesPerRound + bxi;
            uint8_t* rowp = stage + bxi * 4096 + lane * 128;
#pragma unroll
            for (int g = 0; g < 8; ++g)
              *reinterpret_cast<uint4*>(rowp + ((g ^ (lane & 7)) << 4)) =
                  make_uint4(r[c][4 * g], r[c][4 * g + 1], r[c][4 * g + 2], r[c][4 * g + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int bxi = 0; bxi < Cfg::kDqBoxesPerRound; ++bxi)
              // boxes of 32 columns; those wholly past d (D > d) are not sent
              if ((rd * Cfg::kDqBoxesPerRound + bxi) * 32 < p.dcols)
                tma_reduce_add_3d(&tm_dq, (rd * Cfg::kDqBoxesPerRound + bxi) * 32, yz.x, yz.y,
                                  stage_u32 + bxi * 4096);
            bulk_commit_group();
            bulk_wait_group_read0();
          }
          __syncwarp();
        }
        if (*abort_flag) { ok = false; break; }
      }
    }
    if (lane == 0) bulk_wait_group0();
    __syncwarp();
    if (!ok) *abort_flag = 1;
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, Cfg::kTmemCols);
}

}  // namespace fa
