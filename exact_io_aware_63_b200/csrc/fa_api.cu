// fa_api.cu - the C ABI declared in include/fa.h: argument checks, TMA tensor
// map encoding, work-unit counts and kernel launches.  All arithmetic of the
// attention path runs in the kernels of fa_fwd.cuh and fa_bwd.cuh.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_bwd.cuh"
#include "fa_bwd_det.cuh"
#include "fa_d256.cuh"
#include "fa_fwd.cuh"

namespace fa {

// Check of the bounded-wait machinery every kernel relies on: one warp waits
// on a shared-memory mbarrier with the given limit.  With arrive = 0 nothing
// completes the barrier's phase, so the wait must give up, record
// FA_DEV_TIMEOUT in the status word and return; with arrive = 1 the warp
// arrives first and the wait succeeds at once.  Either way the kernel ends.
__global__ void __launch_bounds__(32, 1)
    fa_selftest_wait_kernel(int arrive, unsigned long long limit_ns, int* result) {
  __shared__ __align__(8) unsigned long long bar_storage;
  const uint32_t bar = smem_u32(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  if (arrive && threadIdx.x == 0) mbar_arrive(bar);
  __syncwarp();
  const bool ok = mbar_wait_for(bar, 0, limit_ns);
  if (threadIdx.x == 0) *result = ok ? 1 : 0;
}

// The FMA-pipe exponential of the softmax (ex2_poly, and ex2_poly2 on
// pairs) evaluated element by element, for tests of its error bound.
__global__ void __launch_bounds__(256) fa_selftest_ex2_kernel(const float* __restrict__ x,
                                                              float* __restrict__ y, int n,
                                                              int pair) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (pair) {
    const int i0 = 2 * i, i1 = 2 * i + 1;
    if (i0 >= n) return;
    const float x0 = x[i0], x1 = (i1 < n) ? x[i1] : 0.f;
    float y0, y1;
    ex2_poly2(x0, x1, y0, y1);
    y[i0] = y0;
    if (i1 < n) y[i1] = y1;
  } else if (i < n) {
    y[i] = ex2_poly(x[i]);
  }
}

}  // namespace fa

namespace {

constexpr int kVersion = 10000;  // 1.0.0

// ---------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [B*H][N][d] bf16 tensor viewed per head (x = column, y = row within the
// head, z = head), boxes of 128 rows x 64 columns, 128-byte swizzle.  Rows of
// a box beyond N are zero-filled on loads and dropped on stores, so a partial
// last tile never touches the next head.
// box_rows = 32 gives the row-chunk boxes of the head-dimension-256 kernels.
bool make_tmap(CUtensorMap* m, const void* base, int BH, int N, int d, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// [B*H][N][d] float32 accumulator viewed per head, boxes of 32 rows x 32
// columns (128 bytes), 128-byte swizzle: the target of the dQ TMA reduce-adds.
bool make_tmap_f32_acc(CUtensorMap* m, const void* base, int BH, int N, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N),
                        static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(N) * d * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Packed [T][H][d] tensors (variable-length batches) mapped as (d, H, T), so
// that the strides increase: box (64, 1, 128) is a 128-token tile of one head,
// laid out in shared memory exactly like the (64, 128, 1) box of make_tmap.
bool make_tmap_packed(CUtensorMap* m, const void* base, int H, int T, int d, int box_rows = 128) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The float32 [T][H][d] dQ accumulator of a packed batch: boxes of 32 tokens x
// 32 columns of one head.
bool make_tmap_f32_acc_packed(CUtensorMap* m, const void* base, int H, int T, int d) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(T)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(H) * d * 4};
  cuuint32_t box[3] = {32, 1, 32};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Geometry of a packed variable-length batch (cu == nullptr: the [B][H][N][d]
// layout).  N passed alongside is the longest sequence.
struct Packed {
  const int32_t* cu = nullptr;
  int T = 0;
};

// Tensor map of a bf16 operand in either layout.
bool make_tmap_any(CUtensorMap* m, const void* base, int B, int H, int N, int d, const Packed& pk,
                   int box_rows = 128) {
  return pk.cu ? make_tmap_packed(m, base, H, pk.T, d, box_rows)
               : make_tmap(m, base, B * H, N, d, box_rows);
}

// Launches a kernel with programmatic stream serialization: it may be
// scheduled while the previous kernel in the stream is finishing, and waits
// (griddepcontrol.wait, in the kernel) before it touches global memory.  This
// hides the launch gap between the library's back-to-back kernels.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by every entry point.  Returns FA_OK, an error, or 1
// for "empty problem: nothing to do".
// Head dimensions: 64, 128 and 256 natively; 32 and 96 run on the 64 / 128
// kernels, whose tensor maps read the missing columns as zeros and whose stores
// stop at d.
bool supported_d(int d) { return d == 32 || d == 64 || d == 96 || d == 128 || d == 256; }

int check_shape(int B, int H, int N, int d) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_SHAPE;
  if (!supported_d(d)) return FA_ERR_UNSUPPORTED_D;
  if (B == 0 || H == 0 || N == 0) return 1;
  const long long rows = static_cast<long long>(B) * H * N;
  if (rows >= (1LL << 31)) return FA_ERR_SHAPE;
  return FA_OK;
}

// Checks of a packed variable-length batch (before check_shape, which then
// sees B, H and max_seqlen): FA_OK, an error, or 1 for "nothing to do".
int check_packed(const int32_t* cu, int B, int H, int max_seqlen, int T, int d) {
  if (B < 0 || H < 0 || max_seqlen < 0 || T < 0) return FA_ERR_SHAPE;
  if (!supported_d(d)) return FA_ERR_UNSUPPORTED_D;
  if (B == 0 || H == 0 || max_seqlen == 0 || T == 0) return 1;
  // B sequences of at most max_seqlen tokens: the workspace and the unit grid
  // are sized for B * max_seqlen rows per head
  if (static_cast<long long>(T) > static_cast<long long>(B) * max_seqlen) return FA_ERR_SHAPE;
  if (!cu) return FA_ERR_NULL;
  if (!aligned(cu, 4)) return FA_ERR_ALIGN;
  return FA_OK;
}

int check_scale(float scale) {
  return (std::isfinite(scale) && scale > 0.f) ? FA_OK : FA_ERR_ARG;
}

constexpr int kMaxDevices = 64;  // devices whose per-device state is cached

// Makes the device that owns `ptr` current for this runtime instance and
// returns its SM count (0 on failure).
int select_device(const void* ptr) {
  cudaPointerAttributes attr;
  if (cudaPointerGetAttributes(&attr, ptr) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  int dev = attr.device;
  if (dev < 0) return 0;
  if (cudaSetDevice(dev) != cudaSuccess) return 0;
  static std::atomic<int> sm_count[kMaxDevices];
  if (dev < kMaxDevices) {
    const int cached = sm_count[dev].load(std::memory_order_relaxed);
    if (cached > 0) return cached;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (dev < kMaxDevices) sm_count[dev].store(n, std::memory_order_relaxed);
  return n;
}

// The opt-in to more than 48 KB of dynamic shared memory (cudaFuncSetAttribute)
// holds for the current device only, so each kernel makes it once per device
// of the process; `done` is that kernel's record, one flag per device.
template <typename Kernel>
bool ensure_smem(Kernel k, int bytes, std::atomic<bool> (&done)[kMaxDevices]) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return false;
  if (dev < kMaxDevices && done[dev].load(std::memory_order_acquire)) return true;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  if (dev < kMaxDevices) done[dev].store(true, std::memory_order_release);
  return true;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Heads per work-unit group: as many as keep `bytes_per_head` of re-read data
// within a 96 MB share of the 126 MB L2, with the heads spread evenly over the
// groups (16 heads in groups of at most 5 become four groups of 4, not 5, 5,
// 5, 1).  Large groups matter for causal masks: the longest unit of the last
// group runs alone at the end of the launch unless the group's work per SM
// exceeds it (a 48 MB share left the SMs idle for 14-20% of a causal 8K
// launch).
int heads_per_group(int BH, double bytes_per_head) {
  const double budget = 96.0 * 1024 * 1024;
  int g = static_cast<int>(budget / bytes_per_head);
  g = g < 1 ? 1 : (g > BH ? BH : g);
  const int groups = (BH + g - 1) / g;
  return (BH + groups - 1) / groups;
}

struct WsLayout {
  size_t delta, lse2, dq_acc, counter, total;
};

// D and LSE2 are kept per head in N rounded up to 128 rows (Rp rows in all),
// so that each 128-row tile of them is one aligned 512-byte block
WsLayout ws_layout(int B, int H, int N, int d) {
  const size_t R = static_cast<size_t>(B) * H * N;
  const size_t Np = (static_cast<size_t>(N) + fa::kTile - 1) / fa::kTile * fa::kTile;
  const size_t Rp = static_cast<size_t>(B) * H * Np;
  WsLayout w;
  w.delta = 0;
  w.lse2 = round_up(w.delta + 4 * Rp, 256);
  w.dq_acc = round_up(w.lse2 + 4 * Rp, 256);
  // head dimension 256 sums dQ on chip (no float32 accumulator in memory)
  const size_t acc_bytes = (d == 256) ? 0 : 4 * R * d;
  w.counter = round_up(w.dq_acc + acc_bytes, 256);
  w.total = w.counter + 256;
  return w;
}

// Dropout arguments after validation: the threshold on the 16-bit draws and
// the weight of kept entries (see FwdParams).
struct DropArgs {
  bool on = false;
  fa::DropoutParams dp = {};
};

int make_drop(float p_drop, uint64_t seed, uint32_t offset, DropArgs* d) {
  if (!(p_drop >= 0.f && p_drop < 1.f)) return FA_ERR_ARG;
  d->on = true;
  const uint32_t t = static_cast<uint32_t>(p_drop * 65536.0f);  // exact product, truncated
  d->dp.t_hi = t << 16;
  d->dp.w = 65536.0f / (65536.0f - static_cast<float>(t));
  d->dp.offset = offset;
  // Philox-4x32-10 round keys: the key (low, high word of seed) bumped by the
  // Weyl constants once per round
  uint32_t k0 = static_cast<uint32_t>(seed), k1 = static_cast<uint32_t>(seed >> 32);
  for (int r = 0; r < 10; ++r) {
    d->dp.rk[2 * r] = k0;
    d->dp.rk[2 * r + 1] = k1;
    k0 += 0x9E3779B9u;
    k1 += 0xBB67AE85u;
  }
  return FA_OK;
}

template <typename P>
void set_drop(P& p, const DropArgs& dr) {
  p.drop = dr.dp;
}

template <int D, bool kPair, bool kDrop, bool kPacked = false>
int launch_fwd_mode(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                    const CUtensorMap& to, fa::FwdParams& p, cudaStream_t stream, int num_sms) {
  using Cfg = fa::FwdCfg<D, kPair>;
  static std::atomic<bool> smem_done[kMaxDevices];
  if (!ensure_smem(fa::fa_fwd_kernel<D, kPair, kDrop, kPacked>, Cfg::kSmemBytes, smem_done))
    return FA_ERR_CUDA;
  const int per_head = kPair ? (p.n_t + 1) / 2 : p.n_t;
  p.num_units = p.B * p.H * per_head;
  const int grid = p.num_units < num_sms ? p.num_units : num_sms;
  const cudaError_t e = launch_pdl(fa::fa_fwd_kernel<D, kPair, kDrop, kPacked>, dim3(grid),
                                   dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, tq, tk, tv, to,
                                   p);
  return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Pair mode (two query tiles share each K/V tile) unless a block mask is
// given: random tile masks give two query tiles few key tiles in common, and
// split mode keeps both softmax warpgroups busy on one query tile instead.
template <int D>
int launch_fwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse, int B,
               int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, uint8_t* visited, cudaStream_t stream, int num_sms,
               const DropArgs& dr, const Packed& pk) {
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap_any(&tq, q, B, H, N, d, pk) || !make_tmap_any(&tk, k, B, H, N, d, pk) ||
      !make_tmap_any(&tv, v, B, H, N, d, pk) || !make_tmap_any(&to, o, B, H, N, d, pk))
    return FA_ERR_CUDA;
  fa::FwdParams p;
  p.o = o;
  p.lse = lse;
  p.block_mask = block_mask;
  p.kv_len = kv_len;
  p.visited = visited;
  p.cu_seqlens = pk.cu;
  p.T = pk.T;
  p.o_stride = pk.cu ? static_cast<long long>(H) * d : d;
  p.dcols = d;
  p.B = B;
  p.H = H;
  p.N = N;
  p.n_t = (N + fa::kTile - 1) / fa::kTile;
  p.heads_per_group = heads_per_group(B * H, 4.0 * N * d);  // K and V
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * fa::kLog2e;
  // the launch's work counter: slots are handed out in turn (see g_fwd_work)
  static std::atomic<unsigned int> ticket{0};
  p.counter_slot = static_cast<int>(ticket.fetch_add(1u, std::memory_order_relaxed) %
                                    static_cast<unsigned int>(fa::kFwdCounterSlots));
  set_drop(p, dr);
  if (pk.cu) {  // packed batches have no block mask: pair mode
    if (dr.on) return launch_fwd_mode<D, true, true, true>(tq, tk, tv, to, p, stream, num_sms);
    return launch_fwd_mode<D, true, false, true>(tq, tk, tv, to, p, stream, num_sms);
  }
  if (dr.on) {
    if (block_mask) return launch_fwd_mode<D, false, true>(tq, tk, tv, to, p, stream, num_sms);
    return launch_fwd_mode<D, true, true>(tq, tk, tv, to, p, stream, num_sms);
  }
  if (block_mask) return launch_fwd_mode<D, false, false>(tq, tk, tv, to, p, stream, num_sms);
  return launch_fwd_mode<D, true, false>(tq, tk, tv, to, p, stream, num_sms);
}

template <int D>
int launch_bwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
               const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv, int B,
               int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
               const int32_t* kv_len, void* workspace, uint8_t* visited, cudaStream_t stream,
               int num_sms, unsigned phases, const DropArgs& dr, const Packed& pk) {
  using Cfg = fa::BwdCfg<D>;
  // rows of the dQ accumulator and of dQ (packed: tokens x heads)
  const long long rows =
      pk.cu ? static_cast<long long>(pk.T) * H : static_cast<long long>(B) * H * N;
  const WsLayout wl = ws_layout(B, H, N, d);  // the caller's workspace, sized for d
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* delta = reinterpret_cast<float*>(ws + wl.delta);
  float* lse2 = reinterpret_cast<float*>(ws + wl.lse2);
  float* dq_acc = reinterpret_cast<float*>(ws + wl.dq_acc);
  int* counter = reinterpret_cast<int*>(ws + wl.counter);
  CUtensorMap tq, tk, tv, tdo, tdq, tdk, tdv;
  const int BH = B * H;
  const bool acc_ok = pk.cu ? make_tmap_f32_acc_packed(&tdq, dq_acc, H, pk.T, d)
                            : make_tmap_f32_acc(&tdq, dq_acc, BH, N, d);
  if (!make_tmap_any(&tq, q, B, H, N, d, pk) || !make_tmap_any(&tk, k, B, H, N, d, pk) ||
      !make_tmap_any(&tv, v, B, H, N, d, pk) || !make_tmap_any(&tdo, dout, B, H, N, d, pk) ||
      !acc_ok || !make_tmap_any(&tdk, dk, B, H, N, d, pk, 32) ||
      !make_tmap_any(&tdv, dv, B, H, N, d, pk, 32))  // dK / dV: 32-row boxes, one per warp
    return FA_ERR_CUDA;
  static std::atomic<bool> smem_done[4][kMaxDevices];
  if (!ensure_smem(fa::fa_bwd_kernel<D, false, false>, Cfg::kSmemBytes, smem_done[0]) ||
      !ensure_smem(fa::fa_bwd_kernel<D, true, false>, Cfg::kSmemBytes, smem_done[1]) ||
      !ensure_smem(fa::fa_bwd_kernel<D, false, true>, Cfg::kSmemBytes, smem_done[2]) ||
      !ensure_smem(fa::fa_bwd_kernel<D, true, true>, Cfg::kSmemBytes, smem_done[3]))
    return FA_ERR_CUDA;
  // preprocess
  if (phases & 1u) {
    const int threads = 256;
    const int Np = (N + fa::kTile - 1) / fa::kTile * fa::kTile;
    const long long rows_p = static_cast<long long>(B) * H * Np;
    const long long work = (rows > rows_p ? rows : rows_p) * (D / 4);  // lanes cover D columns
    long long blocks = (work + threads - 1) / threads;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    cudaError_t e;
    if (pk.cu)
      e = launch_pdl(fa::fa_bwd_pre_packed_kernel<D>, dim3(static_cast<int>(blocks)),
                     dim3(threads), 0, stream, o, dout, lse, delta, lse2,
                     reinterpret_cast<float4*>(dq_acc), counter, pk.cu, H, N, Np, pk.T, rows_p,
                     rows, d);
    else
      e = launch_pdl(fa::fa_bwd_pre_kernel<D>, dim3(static_cast<int>(blocks)), dim3(threads), 0,
                     stream, o, dout, lse, delta, lse2, reinterpret_cast<float4*>(dq_acc), counter,
                     N, Np, rows_p, rows, d);
    if (e != cudaSuccess) return FA_ERR_CUDA;
  }
  // main
  if (phases & 2u) {
    fa::BwdParams p;
    p.dq_acc = dq_acc;
    p.delta = delta;
    p.lse2 = lse2;
    p.dk = dk;
    p.dv = dv;
    p.block_mask = block_mask;
    p.kv_len = kv_len;
    p.visited = visited;
    p.cu_seqlens = pk.cu;
    p.T = pk.T;
    p.o_stride = pk.cu ? static_cast<long long>(H) * d : d;
    p.dcols = d;
    p.B = B;
    p.H = H;
    p.N = N;
    p.n_t = (N + fa::kTile - 1) / fa::kTile;
    p.num_units = B * H * p.n_t;
    p.heads_per_group = heads_per_group(B * H, 8.0 * N * d);  // Q, dO, f32 dQ accumulator
    p.work_counter = counter;
    p.causal = causal ? 1 : 0;
    p.scale = scale;
    p.scale_log2 = scale * fa::kLog2e;
    set_drop(p, dr);
    const int grid = p.num_units < num_sms ? p.num_units : num_sms;
    auto kernel = pk.cu ? (dr.on ? fa::fa_bwd_kernel<D, true, true>
                                 : fa::fa_bwd_kernel<D, false, true>)
                        : (dr.on ? fa::fa_bwd_kernel<D, true, false>
                                 : fa::fa_bwd_kernel<D, false, false>);
    if (launch_pdl(kernel, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes, stream, tq, tk, tv,
                   tdo, tdq, tdk, tdv, p) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  // dQ
  if (phases & 4u) {
    const int threads = 256;
    const long long n8 = rows * d / 8;  // dQ is [rows][d]
    long long blocks = (n8 + threads - 1) / threads;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    if (launch_pdl(fa::fa_bwd_dq_kernel, dim3(static_cast<int>(blocks)), dim3(threads), 0, stream,
                   reinterpret_cast<const float4*>(dq_acc), reinterpret_cast<uint4*>(dq), scale,
                   n8) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  // dQ without atomics: one CTA walks each query tile's key tiles in order
  // (head dimensions 64 and 128 only: bwd_impl checks it before any launch)
  if (phases & 8u) {
    using DCfg = fa::DetCfg<D>;
    static std::atomic<bool> det_smem_done[kMaxDevices];
    if (!ensure_smem(fa::fa_bwd_dq_det_kernel<D>, DCfg::kSmemBytes, det_smem_done))
      return FA_ERR_CUDA;
    fa::DetParams dp;
    fa::FwdParams& sp = dp.sched;
    sp.o = nullptr;
    sp.lse = nullptr;
    sp.block_mask = block_mask;
    sp.kv_len = kv_len;
    sp.visited = nullptr;
    sp.cu_seqlens = nullptr;  // the ordered dQ kernel takes the [B][H][N][d] layout only
    sp.T = 0;
    sp.o_stride = D;
    sp.dcols = D;
    sp.B = B;
    sp.H = H;
    sp.N = N;
    sp.n_t = (N + fa::kTile - 1) / fa::kTile;
    sp.num_units = B * H * sp.n_t;
    sp.heads_per_group = heads_per_group(B * H, 4.0 * N * D);  // K and V
    sp.causal = causal ? 1 : 0;
    sp.scale_log2 = scale * fa::kLog2e;
    sp.counter_slot = 0;  // the ordered dQ kernel deals its units statically
    dp.delta = delta;
    dp.lse2 = lse2;
    dp.dq = dq;
    dp.scale = scale;
    const int grid = sp.num_units < num_sms ? sp.num_units : num_sms;
    if (launch_pdl(fa::fa_bwd_dq_det_kernel<D>, dim3(grid), dim3(DCfg::kThreads),
                   DCfg::kSmemBytes, stream, tq, tk, tv, tdo, dp) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  return FA_OK;
}

// Head dimension 256: one query tile per unit (see fa_d256.cuh).
int launch_fwd256(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                  int B, int H, int N, float scale, int causal, const uint8_t* block_mask,
                  const int32_t* kv_len, uint8_t* visited, cudaStream_t stream, int num_sms) {
  using Cfg = fa::Fwd256Cfg;
  const int BH = B * H;
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap(&tq, q, BH, N, 256) || !make_tmap(&tk, k, BH, N, 256) ||
      !make_tmap(&tv, v, BH, N, 256, 32) || !make_tmap(&to, o, BH, N, 256))
    return FA_ERR_CUDA;
  fa::FwdParams p = {};
  p.o = o;
  p.lse = lse;
  p.block_mask = block_mask;
  p.kv_len = kv_len;
  p.visited = visited;
  p.o_stride = 256;
  p.dcols = 256;
  p.B = B;
  p.H = H;
  p.N = N;
  p.n_t = (N + fa::kTile - 1) / fa::kTile;
  p.num_units = BH * p.n_t;
  p.heads_per_group = heads_per_group(BH, 4.0 * N * 256);  // K and V
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * fa::kLog2e;
  static std::atomic<bool> smem_done[kMaxDevices];
  if (!ensure_smem(fa::fa_fwd256_kernel<false>, Cfg::kSmemBytes, smem_done)) return FA_ERR_CUDA;
  const int grid = p.num_units < num_sms ? p.num_units : num_sms;
  return launch_pdl(fa::fa_fwd256_kernel<false>, dim3(grid), dim3(Cfg::kThreads), Cfg::kSmemBytes,
                    stream, tq, tk, tv, to, p) == cudaSuccess
             ? FA_OK
             : FA_ERR_CUDA;
}

// Head dimension 256 backward: preprocess (phase 0), the dK and dV passes
// (phase 1), the dQ pass (phase 2, and phase 3: it is already ordered).
int launch_bwd256(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                  const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                  int B, int H, int N, float scale, int causal, const uint8_t* block_mask,
                  const int32_t* kv_len, void* workspace, uint8_t* visited, cudaStream_t stream,
                  int num_sms, unsigned phases) {
  using Cfg = fa::Bwd256Cfg;
  constexpr int d = 256;
  const int BH = B * H;
  const WsLayout wl = ws_layout(B, H, N, d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* delta = reinterpret_cast<float*>(ws + wl.delta);
  float* lse2 = reinterpret_cast<float*>(ws + wl.lse2);
  int* counter = reinterpret_cast<int*>(ws + wl.counter);
  const int n_t = (N + fa::kTile - 1) / fa::kTile;
  if (phases & 1u) {
    const int threads = 256;
    const long long rows_p = static_cast<long long>(BH) * n_t * fa::kTile;
    long long blocks = (rows_p * (d / 4) + threads - 1) / threads;
    const long long cap = static_cast<long long>(num_sms) * 8;
    if (blocks > cap) blocks = cap;
    // no dQ accumulator to zero (rows = 0)
    if (launch_pdl(fa::fa_bwd_pre_kernel<256>, dim3(static_cast<int>(blocks)), dim3(threads), 0,
                   stream, o, dout, lse, delta, lse2, static_cast<float4*>(nullptr), counter, N,
                   n_t * fa::kTile, rows_p, 0ll, d) != cudaSuccess)
      return FA_ERR_CUDA;
  }
  if (!(phases & 14u)) return FA_OK;
  CUtensorMap tq, tk, tv, tdo, tq32, tk32, tdo32, tdq, tdk, tdv;
  if (!make_tmap(&tq, q, BH, N, d) || !make_tmap(&tk, k, BH, N, d) ||
      !make_tmap(&tv, v, BH, N, d) || !make_tmap(&tdo, dout, BH, N, d) ||
      !make_tmap(&tq32, q, BH, N, d, 32) || !make_tmap(&tk32, k, BH, N, d, 32) ||
      !make_tmap(&tdo32, dout, BH, N, d, 32) || !make_tmap(&tdq, dq, BH, N, d) ||
      !make_tmap(&tdk, dk, BH, N, d) || !make_tmap(&tdv, dv, BH, N, d))
    return FA_ERR_CUDA;
  fa::Bwd256Params bp = {};
  fa::FwdParams& pq = bp.q;
  pq.block_mask = block_mask;
  pq.kv_len = kv_len;
  pq.visited = visited;
  pq.o_stride = d;
  pq.dcols = d;
  pq.B = B;
  pq.H = H;
  pq.N = N;
  pq.n_t = n_t;
  pq.num_units = BH * n_t;
  pq.heads_per_group = heads_per_group(BH, 4.0 * N * d);  // K and V
  pq.causal = causal ? 1 : 0;
  pq.scale_log2 = scale * fa::kLog2e;
  fa::BwdParams& pk = bp.k;
  pk.delta = delta;
  pk.lse2 = lse2;
  pk.dk = dk;
  pk.dv = dv;
  pk.block_mask = block_mask;
  pk.kv_len = kv_len;
  pk.visited = visited;
  pk.o_stride = d;
  pk.dcols = d;
  pk.B = B;
  pk.H = H;
  pk.N = N;
  pk.n_t = n_t;
  pk.num_units = BH * n_t;
  pk.heads_per_group = heads_per_group(BH, 4.0 * N * d);  // Q and dO
  pk.work_counter = counter;
  pk.causal = causal ? 1 : 0;
  pk.scale = scale;
  pk.scale_log2 = scale * fa::kLog2e;
  bp.dq = dq;
  static std::atomic<bool> smem_done[3][kMaxDevices];
  if (!ensure_smem(fa::fa_bwd256_kernel<fa::kPassDQ>, Cfg::kSmemBytes, smem_done[0]) ||
      !ensure_smem(fa::fa_bwd256_kernel<fa::kPassDK>, Cfg::kSmemBytes, smem_done[1]) ||
      !ensure_smem(fa::fa_bwd256_kernel<fa::kPassDV>, Cfg::kSmemBytes, smem_done[2]))
    return FA_ERR_CUDA;
  const int grid = pk.num_units < num_sms ? pk.num_units : num_sms;
  if (phases & 2u) {
    if (launch_pdl(fa::fa_bwd256_kernel<fa::kPassDK>, dim3(grid), dim3(Cfg::kThreads),
                   Cfg::kSmemBytes, stream, tq, tk, tv, tdo, tq32, tk32, tdo32, tdk, bp) !=
            cudaSuccess ||
        launch_pdl(fa::fa_bwd256_kernel<fa::kPassDV>, dim3(grid), dim3(Cfg::kThreads),
                   Cfg::kSmemBytes, stream, tq, tk, tv, tdo, tq32, tk32, tdo32, tdv, bp) !=
            cudaSuccess)
      return FA_ERR_CUDA;
  }
  if (phases & 12u) {
    if (launch_pdl(fa::fa_bwd256_kernel<fa::kPassDQ>, dim3(grid), dim3(Cfg::kThreads),
                   Cfg::kSmemBytes, stream, tq, tk, tv, tdo, tq32, tk32, tdo32, tdq, bp) !=
        cudaSuccess)
      return FA_ERR_CUDA;
  }
  return FA_OK;
}

int fwd_impl(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse, int B,
             int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
             const int32_t* kv_len, uint8_t* visited, void* stream,
             const DropArgs& dr = DropArgs(), const Packed& pk = Packed()) {
  int rc = check_shape(B, H, N, d);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (d == 256 && (dr.on || pk.cu)) return FA_ERR_UNSUPPORTED_D;  // no dropout / packed form
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGN;
  if (kv_len && !aligned(kv_len, 4)) return FA_ERR_ALIGN;
  rc = check_scale(scale);
  if (rc != FA_OK) return rc;
  const int sms = select_device(q);
  if (sms <= 0) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256)
    return launch_fwd256(q, k, v, o, lse, B, H, N, scale, causal, block_mask, kv_len, visited, s,
                         sms);
  if (d <= 64)
    return launch_fwd<64>(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, visited,
                          s, sms, dr, pk);
  return launch_fwd<128>(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, visited,
                         s, sms, dr, pk);
}

int bwd_impl(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
             const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv, int B,
             int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
             const int32_t* kv_len, void* workspace, size_t workspace_bytes, uint8_t* visited,
             void* stream, unsigned phases = 7u, const DropArgs& dr = DropArgs(),
             const Packed& pk = Packed()) {
  int rc = check_shape(B, H, N, d);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if ((phases & 8u) && d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED_D;  // ordered dQ
  if (d == 256 && (dr.on || pk.cu)) return FA_ERR_UNSUPPORTED_D;  // no dropout / packed form
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      !aligned(dout, 16) || !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
      !aligned(lse, 4))
    return FA_ERR_ALIGN;
  if (kv_len && !aligned(kv_len, 4)) return FA_ERR_ALIGN;
  rc = check_scale(scale);
  if (rc != FA_OK) return rc;
  if (!workspace || workspace_bytes < ws_layout(B, H, N, d).total) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return FA_ERR_ALIGN;
  const int sms = select_device(q);
  if (sms <= 0) return FA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (d == 256)
    return launch_bwd256(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, scale, causal, block_mask,
                         kv_len, workspace, visited, s, sms, phases);
  if (d <= 64)
    return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                          block_mask, kv_len, workspace, visited, s, sms, phases, dr, pk);
  return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal,
                         block_mask, kv_len, workspace, visited, s, sms, phases, dr, pk);
}

}  // namespace

extern "C" {

int fa_fwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse, int B,
           int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
           const int32_t* kv_len, void* stream) {
  return fwd_impl(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, nullptr, stream);
}

int fa_fwd_traced(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                  int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                  const int32_t* kv_len, uint8_t* visited, void* stream) {
  if (!visited && B > 0 && H > 0 && N > 0) return FA_ERR_NULL;
  return fwd_impl(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, visited, stream);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  const int rc = check_shape(B, H, N, d);
  if (rc != FA_OK) return 0;
  return ws_layout(B, H, N, d).total;
}

int fa_bwd(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
           const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv, int B,
           int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
           const int32_t* kv_len, void* workspace, size_t workspace_bytes, void* stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, nullptr, stream);
}

int fa_bwd_traced(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                  const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                  int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                  const int32_t* kv_len, void* workspace, size_t workspace_bytes,
                  uint8_t* visited, void* stream) {
  if (!visited && B > 0 && H > 0 && N > 0) return FA_ERR_NULL;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, visited, stream);
}

int fa_bwd_phase(int phase, const fa_bf16* q, const fa_bf16* k, const fa_bf16* v,
                 const fa_bf16* o, const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk,
                 fa_bf16* dv, int B, int H, int N, int d, float scale, int causal,
                 const uint8_t* block_mask, const int32_t* kv_len, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (phase < 0 || phase > 3) return FA_ERR_ARG;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, nullptr, stream, 1u << phase);
}

int fa_bwd_deterministic(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                         const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk,
                         fa_bf16* dv, int B, int H, int N, int d, float scale, int causal,
                         const uint8_t* block_mask, const int32_t* kv_len, void* workspace,
                         size_t workspace_bytes, void* stream) {
  // preprocess, main kernel (its dK and dV), then dQ by the ordered kernel
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, nullptr, stream, 1u | 2u | 8u);
}

int fa_fwd_dropout(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                   const int32_t* kv_len, float p_drop, uint64_t seed, uint32_t offset,
                   void* stream) {
  DropArgs dr;
  const int rc = make_drop(p_drop, seed, offset, &dr);
  if (rc != FA_OK) return rc;
  return fwd_impl(q, k, v, o, lse, B, H, N, d, scale, causal, block_mask, kv_len, nullptr, stream,
                  dr);
}

int fa_bwd_dropout(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                   const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* block_mask,
                   const int32_t* kv_len, float p_drop, uint64_t seed, uint32_t offset,
                   void* workspace, size_t workspace_bytes, void* stream) {
  DropArgs dr;
  const int rc = make_drop(p_drop, seed, offset, &dr);
  if (rc != FA_OK) return rc;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  workspace, workspace_bytes, nullptr, stream, 7u, dr);
}

int fa_selftest_wait_timeout(int arrive, unsigned int limit_us, int* result, void* stream) {
  if (!result) return FA_ERR_NULL;
  if (!aligned(result, 4)) return FA_ERR_ALIGN;
  if (limit_us == 0 || limit_us > 2000000u) return FA_ERR_ARG;
  fa::fa_selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      arrive ? 1 : 0, 1000ull * limit_us, result);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_selftest_ex2(const float* x, float* y, int n, int pair, void* stream) {
  if (n < 0) return FA_ERR_SHAPE;
  if (n == 0) return FA_OK;
  if (!x || !y) return FA_ERR_NULL;
  if (!aligned(x, 4) || !aligned(y, 4)) return FA_ERR_ALIGN;
  const long long threads = pair ? (static_cast<long long>(n) + 1) / 2 : n;
  const int blocks = static_cast<int>((threads + 255) / 256);
  fa::fa_selftest_ex2_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, y, n, pair ? 1 : 0);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_fwd_varlen(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, fa_bf16* o, float* lse,
                  const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total_tokens, int d,
                  float scale, int causal, float p_drop, uint64_t seed, uint32_t offset,
                  void* stream) {
  DropArgs dr;
  int rc = make_drop(p_drop, seed, offset, &dr);
  if (rc != FA_OK) return rc;
  if (p_drop == 0.f) dr = DropArgs();  // keep-all: the kernels without dropout
  rc = check_packed(cu_seqlens, B, H, max_seqlen, total_tokens, d);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  Packed pk;
  pk.cu = cu_seqlens;
  pk.T = total_tokens;
  return fwd_impl(q, k, v, o, lse, B, H, max_seqlen, d, scale, causal, nullptr, nullptr, nullptr,
                  stream, dr, pk);
}

int fa_bwd_varlen(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v, const fa_bf16* o,
                  const float* lse, const fa_bf16* dout, fa_bf16* dq, fa_bf16* dk, fa_bf16* dv,
                  const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total_tokens, int d,
                  float scale, int causal, float p_drop, uint64_t seed, uint32_t offset,
                  void* workspace, size_t workspace_bytes, void* stream) {
  DropArgs dr;
  int rc = make_drop(p_drop, seed, offset, &dr);
  if (rc != FA_OK) return rc;
  if (p_drop == 0.f) dr = DropArgs();
  rc = check_packed(cu_seqlens, B, H, max_seqlen, total_tokens, d);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  Packed pk;
  pk.cu = cu_seqlens;
  pk.T = total_tokens;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, max_seqlen, d, scale, causal, nullptr,
                  nullptr, workspace, workspace_bytes, nullptr, stream, 7u, dr, pk);
}

int fa_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_device_status, sizeof(v)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const unsigned int z = 0;
    if (cudaMemcpyToSymbol(fa::g_device_status, &z, sizeof(z)) != cudaSuccess) return FA_ERR_CUDA;
    return (v & fa::FA_DEV_TIMEOUT) ? FA_ERR_TIMEOUT : FA_ERR_CUDA;
  }
  return FA_OK;
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "a required pointer is NULL";
    case FA_ERR_ALIGN: return "a pointer is not aligned as required";
    case FA_ERR_SHAPE: return "unsupported shape (negative size, or B*H*N >= 2^31)";
    case FA_ERR_UNSUPPORTED_D:
      return "head dimension d must be 32, 64, 96, 128 or 256 (64, 128 or 256 for the ordered "
             "dQ; 256 has no dropout or packed form)";
    case FA_ERR_WORKSPACE: return "workspace missing or smaller than fa_bwd_workspace_size()";
    case FA_ERR_CUDA: return "a CUDA runtime or driver call failed";
    case FA_ERR_TIMEOUT: return "a device pipeline wait timed out; outputs are incomplete";
    case FA_ERR_ARG:
      return "invalid argument (scale not finite or not > 0, unknown phase, or dropout "
             "probability outside [0, 1))";
    case FA_ERR_SCRATCH_LIMIT:
      return "shape needs more backward scratch than the built-in FA_BWD_NOALLOC_SCRATCH_BYTES";
    default: return "unknown status";
  }
}

int fa_version(void) { return kVersion; }

}  // extern "C"

// ---------------------------------------------------------------------------
// fa_bwd_noalloc: the backward pass with its scratch in a static device array,
// for callers that cannot allocate device memory.  The array is the whole
// workspace of fa_bwd (same layout); kernels receive its device address as
// an ordinary pointer.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char fa_bwd_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};
unsigned long long g_noalloc_ctx[kMaxDevices] = {};  // context the address belongs to

// Process-unique id of the calling thread's current CUDA context (0 if the
// driver cannot tell).  A device reset replaces the context, and with it the
// module and the array's address; the new context has a new id.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(ptr);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of fa_bwd_noalloc_scratch on the current device `dev`, looked
// up once per device (again only if the device's context has been replaced,
// as by cudaDeviceReset) and cached.  In host code the array's name is only a
// host-side handle, never a usable device address.
int noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  // the caller has made `dev` current with cudaSetDevice, which also binds its
  // primary context to this thread
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> guard(g_noalloc_mutex);
  if (!g_noalloc_ptr[dev] || ctx == 0 || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, fa_bwd_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return FA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

extern "C" int fa_bwd_noalloc(const fa_bf16* q, const fa_bf16* k, const fa_bf16* v,
                              const fa_bf16* o, const float* lse, const fa_bf16* dout,
                              fa_bf16* dq, fa_bf16* dk, fa_bf16* dv, int B, int H, int N, int d,
                              float scale, int causal, const uint8_t* block_mask,
                              const int32_t* kv_len, void* stream) {
  int rc = check_shape(B, H, N, d);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  const size_t need = ws_layout(B, H, N, d).total;
  if (need > static_cast<size_t>(FA_BWD_NOALLOC_SCRATCH_BYTES)) return FA_ERR_SCRATCH_LIMIT;
  if (!q) return FA_ERR_NULL;
  if (!aligned(q, 16)) return FA_ERR_ALIGN;
  if (select_device(q) <= 0) return FA_ERR_CUDA;  // makes q's device current
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  void* scratch = nullptr;
  rc = noalloc_scratch(dev, &scratch);
  if (rc != FA_OK) return rc;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, block_mask, kv_len,
                  scratch, static_cast<size_t>(FA_BWD_NOALLOC_SCRATCH_BYTES), nullptr, stream);
}
