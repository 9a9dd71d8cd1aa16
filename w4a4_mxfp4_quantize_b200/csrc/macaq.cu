// B200 (sm_100a) MACAQ W4A4 MXFP4 linear: kernels and the C ABI of macaq.h.
//
// Data layout.  Both MMA operands live in "tile images": 128 rows x 256 K
// elements, E2M1 codes in 128-byte rows with the 128-byte XOR swizzle the
// tensor core's K-major shared-memory descriptor expects (16384 bytes), plus a
// 1024-byte E8M0 scale image in the order tcgen05.cp copies into tensor
// memory.  Offline weights are stored as such images; activations are either
// quantised straight into shared memory (fused path) or quantised once into
// images in an L2-resident workspace (quantise-once path).
//
// Small M (fused kernel): the MMA is swapped, operand A = 128 output channels of
// weights (the MMA's M side), operand B = a tile of BT tokens (its N side,
// 16..128), so the token count maps to the narrow side of tcgen05.mma and
// D[n][t] sits in TMEM with one output channel per lane.  Large M (GEMM): A = a
// 128-token activation tile, B = 256 output channels (two weight images), one
// token per TMEM lane.
//
// Kernels
//   calibrate_kernel      offline: channel factors D from calibration rows and W
//   prep_weights_kernel   offline: W*D -> FWHT32 -> MX -> weight tile images
//   quant_tiles_kernel    activation prologue over all rows once -> tile images
//                         (dense rows, or group-padded rows for the grouped form;
//                         only 32-row slabs that hold rows)
//   group_tables_kernel   grouped: validate group_list; row offsets, tile prefix,
//                         experts and the quantiser's slab table
//   gemm_kernel           persistent, warp-specialised tcgen05 kind::mxf4 GEMM
//                         over tile images, 128 x 256 output tiles, one TMEM
//                         accumulator drained to registers, epilogue staged in
//                         shared memory and stored as coalesced row runs;
//                         chained to the quantiser by programmatic dependent
//                         launch
//   fused_small_kernel    small M: one kernel, the activation prologue writes
//                         the swizzled B tile straight into shared memory;
//                         optional split-K across a thread-block cluster, partial
//                         sums reduced through distributed shared memory
//   quant_canonical_kernel, export_tiles_kernel, mx_encode_kernel: tests only
#include <cuda_runtime.h>

#include <cmath>
#include <algorithm>
#include <cstdint>
#include <cstring>
#include <utility>
#include <vector>

#include "macaq.h"
#include "mx.cuh"
#include "ptx.cuh"

namespace macaq {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bounded waits give up after 2 s
constexpr int kMaxGroups = 1024;
constexpr size_t kWsReserved = 4096;  // first bytes of every workspace, left untouched
constexpr int kSmallM = 128;          // dense calls up to this many rows use the fused kernel

__host__ __device__ constexpr int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint16_t bf16_bits(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

// Output activation of npu_grouped_matmul's act_type (parameter act_type: 0 none,
// 1 RELU, 2 GELU_TANH, 4 FAST_GELU, 5 SILU), in FP32.  The three gated forms are
// v * sigmoid(a) with a = 2u, u = sqrt(2/pi) (v + 0.044715 v^3) for GELU_TANH
// (0.5 (1 + tanh u) = sigmoid(2u)), a = 1.702 v for FAST_GELU (named on the page
// without a formula), a = v for SILU, and are evaluated as
//   v sigmoid(a) = h + h tanh(a / 2),  h = v / 2,
// with tanh taken in half precision by the hardware (tanh_h: the argument rounded
// to FP16, relative error of the approximation about 2^-11) and no division.
// The error in y is at most about 5e-4 |v|, far below the MXFP4 quantisation
// noise of v.  The form needs one special-function operation per two outputs;
// an exponential plus a reciprocal per output (two such operations, at 16 per
// clock per SM) alone took about twice the tensor core's time for a 128 x 256
// tile at K = 1024.  act_value (one output) and act_pair (two, in packed FP32
// pair instructions) take the same steps and give the same bits.
constexpr float kGeluC0 = 0.7978845608028654f;    // sqrt(2/pi)
constexpr float kGeluC1 = 0.035677408136300125f;  // sqrt(2/pi) x 0.044715
constexpr float kFastGeluHalf = 0.851f;           // 1.702 / 2
template <int ACT>
__device__ __forceinline__ float act_value(float v) {
  if constexpr (ACT == 1) {
    return fmaxf(v, 0.f);
  } else if constexpr (ACT == 2) {
    const float u = v * fmaf(v * v, kGeluC1, kGeluC0);
    const float h = 0.5f * v;
    return fmaf(h, tanh_h(u), h);
  } else if constexpr (ACT == 4) {
    const float h = 0.5f * v;
    return fmaf(h, tanh_h(kFastGeluHalf * v), h);
  } else if constexpr (ACT == 5) {
    const float h = 0.5f * v;
    return fmaf(h, tanh_h(h), h);
  } else {
    return v;
  }
}
template <int ACT>
__device__ __forceinline__ float2 act_pair(float2 v) {
  const float2 half = make_float2(0.5f, 0.5f);
  if constexpr (ACT == 1) {
    return make_float2(fmaxf(v.x, 0.f), fmaxf(v.y, 0.f));
  } else if constexpr (ACT == 2) {
    const float2 u = fmul2(v, ffma2(fmul2(v, v), make_float2(kGeluC1, kGeluC1), make_float2(kGeluC0, kGeluC0)));
    const float2 h = fmul2(v, half);
    return ffma2(h, tanh_h2(u), h);
  } else if constexpr (ACT == 4) {
    const float2 h = fmul2(v, half);
    return ffma2(h, tanh_h2(fmul2(v, make_float2(kFastGeluHalf, kFastGeluHalf))), h);
  } else if constexpr (ACT == 5) {
    const float2 h = fmul2(v, half);
    return ffma2(h, tanh_h2(h), h);
  } else {
    return v;
  }
}
__device__ __forceinline__ float act_value_rt(float v, int act) {
  switch (act) {
    case 1: return act_value<1>(v);
    case 2: return act_value<2>(v);
    case 4: return act_value<4>(v);
    case 5: return act_value<5>(v);
    default: return v;
  }
}

// ============================================================================
// Image layouts
// ============================================================================
// Weights: 128-row x 256-K images (codes 16384 bytes, scales 1024) in pairs, so
// the 256 rows of a wide GEMM tile are one contiguous run per K tile: image
// (e, nt, kt) is number ((e * NT2 + nt / 2) * KT + kt) * 2 + nt % 2, with
// NT2 = ceil(NT / 2) pairs per expert (an odd NT leaves a zero image).
__host__ __device__ __forceinline__ size_t weight_image(int e, int nt, int kt, int NT2, int KT) {
  return ((static_cast<size_t>(e) * NT2 + (nt >> 1)) * KT + kt) * 2 + (nt & 1);
}
// Activations (workspace): per (row tile, K tile) one image of codes followed by
// its scales, so a stage's activation operand is a single copy.
constexpr int kActImageBytes = kTileCodeBytes + kTileSfBytes;  // 17408

// ============================================================================
// Offline weight preparation and test-only kernels
// ============================================================================
// CTA = 32 rows x one 256-wide K tile (256 threads, one 32-block each).
// kPlain: plain MXFP4 of W itself (no D, no Hadamard; D is not read).
// kTrans: W is stored transposed, [E, K, N] (element (n, k) at (e K + k) N + n).
template <bool kPlain, bool kTrans = false>
__global__ void __launch_bounds__(256) prep_weights_kernel(const float* __restrict__ W, const float* __restrict__ D,
                                                           uint8_t* __restrict__ Wq, uint8_t* __restrict__ Ws,
                                                           int N, int K, int NT) {
  // NT: 128-row images per expert including an odd NT's zero image (2 * NT2)
  const int KT = K / kKTile;
  const int kt = blockIdx.y;
  const int t = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int row_global = blockIdx.x * 32 + t;  // over E * NT * 128 padded rows
  const int e = row_global / (NT * kRowsTile);
  const int n = row_global % (NT * kRowsTile);
  const int nt = n / kRowsTile, r = n % kRowsTile;
  const int64_t k0 = static_cast<int64_t>(kt) * kKTile + c * kBlk;
  uint4 codes = make_uint4(0, 0, 0, 0);
  uint32_t scale = 0;
  if (n < N) {
    float wv[32];
    if constexpr (kTrans) {
      const float* wp = W + (static_cast<int64_t>(e) * K + k0) * N + n;  // offline: strided reads are fine
#pragma unroll
      for (int i = 0; i < 32; ++i) wv[i] = __ldg(wp + static_cast<int64_t>(i) * N);
    } else {
      const float4* wp = reinterpret_cast<const float4*>(W + (static_cast<int64_t>(e) * N + n) * K + k0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 a = __ldg(wp + i);
        wv[4 * i] = a.x; wv[4 * i + 1] = a.y; wv[4 * i + 2] = a.z; wv[4 * i + 3] = a.w;
      }
    }
    if constexpr (kPlain) {
      mx_encode_block(wv, codes, scale);
    } else {
      float dv[32];
      const float4* dp = reinterpret_cast<const float4*>(D + static_cast<int64_t>(e) * K + k0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 b = __ldg(dp + i);
        dv[4 * i] = b.x; dv[4 * i + 1] = b.y; dv[4 * i + 2] = b.z; dv[4 * i + 3] = b.w;
      }
      weight_block(wv, dv, codes, scale);
    }
  }
  const size_t tile = weight_image(e, nt, kt, NT / 2, KT);
  *reinterpret_cast<uint4*>(Wq + tile * kTileCodeBytes + code_chunk_offset(r, c)) = codes;
  Ws[tile * kTileSfBytes + sf_offset(r, c)] = static_cast<uint8_t>(scale);
}

// Weight images -> canonical row-major codes/scales (tests only); RT = NT2.
__global__ void __launch_bounds__(256) export_tiles_kernel(const uint8_t* __restrict__ Tq,
                                                           const uint8_t* __restrict__ Ts,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                           int R, int K, int RT, int rows_total) {
  const int KT = K / kKTile;
  const int kt = blockIdx.y;
  const int t = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int row_global = blockIdx.x * 32 + t;  // over E * R
  if (row_global >= rows_total) return;
  const int e = row_global / R, n = row_global % R;
  const int nt = n / kRowsTile, r = n % kRowsTile;
  const size_t tile = weight_image(e, nt, kt, RT, KT);
  const uint4 v = *reinterpret_cast<const uint4*>(Tq + tile * kTileCodeBytes + code_chunk_offset(r, c));
  const uint8_t s = Ts[tile * kTileSfBytes + sf_offset(r, c)];
  const int64_t row = static_cast<int64_t>(e) * R + n;
  *reinterpret_cast<uint4*>(codes + row * (K / 2) + (kt * kKTile + c * kBlk) / 2) = v;
  scales[row * (K / kBlk) + kt * (kKTile / kBlk) + c] = s;
}

// Activation prologue to canonical [M, K/2] codes and [M, K/32] scales (tests).
__global__ void __launch_bounds__(256) quant_canonical_kernel(const uint16_t* __restrict__ x,
                                                              const float* __restrict__ D,
                                                              uint8_t* __restrict__ codes,
                                                              uint8_t* __restrict__ scales, int M, int K) {
  __shared__ __align__(16) float r[kQRcpTile];
  const int kt = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(kt) * kKTile;
  const int t = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int m = blockIdx.x * 32 + t;
  uint4 xv[4] = {};
  if (m < M) {  // issue the activation loads before the reciprocals
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k0 + c * kBlk);
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = __ldg(src + i);
  }
  r[qrcp_index(threadIdx.x)] = __frcp_rn(__ldg(D + k0 + threadIdx.x));
  __syncthreads();
  if (m >= M) return;
  uint4 cv;
  uint32_t sc;
  float2 r2[16];
  load_rcp_block(r + c * kQRcpStride, r2);
  act_block(xv, r2, cv, sc);
  *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(m) * (K / 2) + (k0 + c * kBlk) / 2) = cv;
  scales[static_cast<int64_t>(m) * (K / kBlk) + k0 / kBlk + c] = static_cast<uint8_t>(sc);
}

// MX encoding of raw fp32 blocks (tests the conversion instructions).
__global__ void mx_encode_kernel(const float* __restrict__ v, uint8_t* __restrict__ codes,
                                 uint8_t* __restrict__ scales, int64_t nblocks) {
  const int64_t b = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x;
  if (b >= nblocks) return;
  float u[32];
  const float4* p = reinterpret_cast<const float4*>(v + b * 32);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float4 a = p[i];
    u[4 * i] = a.x; u[4 * i + 1] = a.y; u[4 * i + 2] = a.z; u[4 * i + 3] = a.w;
  }
  uint4 cv;
  uint32_t sc;
  mx_encode_block(u, cv, sc);
  *reinterpret_cast<uint4*>(codes + b * 16) = cv;
  scales[b] = static_cast<uint8_t>(sc);
}

// The bounded wait of the kernels run out on purpose (tests).  One CTA of two
// warps: warp 0 waits on an mbarrier that nothing ever arrives on, with the
// kernels' own bounded wait (mbar_wait) and a limit of timeout_ns; when it gives
// up it raises the CTA's abort flag, and warp 1's wait on the same barrier then
// gives up at the flag (its own limit is the same, as a bound only).  Nothing asynchronous (no
// bulk copy, no tensor-core operation) is issued, so nothing is in flight when
// the waits end.  Thread 0 then reports the expiry to *status the way the
// kernels do.
__global__ void __launch_bounds__(64) wait_expiry_kernel(uint64_t timeout_ns, int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  __shared__ int gave_up[2];
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) gave_up[0] = mbar_wait(&bar, 0, &abort_flag, timeout_ns) ? 0 : 1;
  __syncthreads();
  if (threadIdx.x == 32) gave_up[1] = mbar_wait(&bar, 0, &abort_flag, timeout_ns) ? 0 : 1;
  __syncthreads();
  if (threadIdx.x == 0 && status)
    *status = (abort_flag && gave_up[0] && gave_up[1]) ? MACAQ_ERR_DEVICE_TIMEOUT : MACAQ_OK;
}

// ============================================================================
// Grouped form: device-side group_list validation and tables
// ============================================================================
// Block-wide exclusive scans of three int64 per thread at once (blockDim.x a
// multiple of 32, at most 1024): one pass of warp shuffles, one exchange of the
// warp totals through shared memory.  tot receives the three block totals.
__device__ __forceinline__ void block_excl_scan3(const int64_t (&v)[3], int64_t (&res)[3], int64_t (&tot)[3],
                                                 int64_t* scratch /* [32][3] + [32][3] */) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int64_t inc[3] = {v[0], v[1], v[2]};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int64_t u = __shfl_up_sync(0xffffffffu, inc[i], o);
      if (lane >= o) inc[i] += u;
    }
  }
  if (lane == 31)
    for (int i = 0; i < 3; ++i) scratch[warp * 3 + i] = inc[i];
  __syncthreads();
  // every warp scans the warp totals itself (no second barrier round)
  int64_t wi[3];
#pragma unroll
  for (int i = 0; i < 3; ++i) wi[i] = lane < nw ? scratch[lane * 3 + i] : 0;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
    for (int i = 0; i < 3; ++i) {
      const int64_t u = __shfl_up_sync(0xffffffffu, wi[i], o);
      if (lane >= o) wi[i] += u;
    }
  }
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int64_t before = warp > 0 ? __shfl_sync(0xffffffffu, wi[i], warp - 1) : 0;  // totals of earlier warps
    res[i] = before + inc[i] - v[i];
    tot[i] = __shfl_sync(0xffffffffu, wi[i], nw - 1);
  }
}

// One CTA of 32 * ceil(E / 32) threads, thread g owns group g.  Rules (npu_grouped_matmul,
// group_list / group_list_type): type 0 non-negative and non-decreasing
// cumulative sums, type 1 non-negative counts; the rows must total M.
// Writes goff[0..E] (row offsets), gtp[0..E] (prefix of 128-row tiles per
// list entry), gexp[0..E) (the expert of each entry: the entry itself for types
// 0 and 1, the named group index for type 2), the slab table for the quantiser
// (per 32-row slab holding rows: {expert, first row of x, rows, 4 * tile +
// quarter of the tile}), its length *nslabs and *valid; on a violation also
// *status.
// Weight-list calls (one weight tensor per expert) also pass the device tables
// of the experts' code and scale images; each pointer must be non-null,
// 16-byte aligned (the bulk copies read from it) and must not overlap y, else
// the call is refused on the device with *status set (MACAQ_ERR_NULL, _ALIGN,
// _ALIAS) and y left as it was.
struct WeightList {
  const uint64_t* wq;  // [E] device addresses of the experts' code images (nullptr: stacked weights)
  const uint64_t* ws;  // [E] and of their scale images
  uint64_t wq_bytes, ws_bytes;  // bytes of one expert's images
  uint64_t y_lo, y_hi;          // the output's byte range
};

__global__ void __launch_bounds__(1024) group_tables_kernel(const int64_t* __restrict__ gl, int type, int E, int M,
                                                            int64_t* __restrict__ goff, int* __restrict__ gtp,
                                                            int* __restrict__ gexp, int4* __restrict__ slabs,
                                                            int* __restrict__ nslabs, int* __restrict__ valid,
                                                            int32_t* status, const WeightList wl) {
  __shared__ int64_t scratch[96];
  __shared__ int list_err;
  const int g = threadIdx.x;
  pdl_trigger();  // the quantiser may set up; it reads the tables only after this kernel completes
  int64_t cnt = 0;
  bool bad = false;
  if (g == 0) list_err = 0;
  __syncthreads();
  if (wl.wq != nullptr && g < E) {
    const uint64_t a = wl.wq[g], b = wl.ws[g];
    int err = 0;
    if (a == 0 || b == 0) err = MACAQ_ERR_NULL;
    else if ((a | b) & 15u) err = MACAQ_ERR_ALIGN;
    else if ((a < wl.y_hi && wl.y_lo < a + wl.wq_bytes) || (b < wl.y_hi && wl.y_lo < b + wl.ws_bytes))
      err = MACAQ_ERR_ALIAS;
    if (err != 0) atomicCAS(&list_err, 0, err);
  }
  __syncthreads();
  int ex = g;  // the expert whose weights this list entry's rows use
  if (g < E) {
    if (type == 2) {  // [E, 2] rows of (group index, group size)
      ex = static_cast<int>(gl[2 * g] < 0 || gl[2 * g] >= E ? -1 : gl[2 * g]);
      cnt = gl[2 * g + 1];
      bad = ex < 0 || cnt < 0 || cnt > M;
    } else {
      const int64_t v = gl[g];
      const int64_t prev = (type == 0 && g > 0) ? gl[g - 1] : 0;
      cnt = type == 0 ? v - prev : v;
      bad = v < 0 || cnt < 0 || cnt > M;
    }
  }
  bad = __syncthreads_or(bad);
  if (!bad) {
    const int64_t v[3] = {cnt, (cnt + kRowsTile - 1) / kRowsTile, (cnt + 31) / 32};
    int64_t pre[3], tot[3];
    block_excl_scan3(v, pre, tot, scratch);
    const int64_t rb = pre[0], tb = pre[1], sb = pre[2];
    const int64_t rows_total = tot[0], tiles_total = tot[1], slabs_total = tot[2];
    bad = rows_total != M;
    if (g < E) {
      goff[g] = rb;
      gtp[g] = static_cast<int>(tb);
      gexp[g] = ex;
    }
    if (g == 0) {
      goff[E] = rows_total;
      gtp[E] = static_cast<int>(tiles_total);
      *nslabs = static_cast<int>(slabs_total);
    }
    // slab j of this entry: rows [rb + 32 j, ...) of x, quarter j % 4 of tile tb + j / 4
    if (g < E && !bad)
      for (int64_t j = 0; j * 32 < cnt; ++j)
        slabs[sb + j] = make_int4(ex, static_cast<int>(rb + 32 * j),
                                  static_cast<int>(cnt - 32 * j < 32 ? cnt - 32 * j : 32), static_cast<int>(4 * tb + j));
  }
  if (g == 0) {
    *valid = (bad || list_err != 0) ? 0 : 1;
    if (status && list_err != 0) *status = list_err;
    else if (bad && status) *status = MACAQ_ERR_GROUP_LIST_INVALID;
  }
}

__device__ __forceinline__ int find_group(const int* gtp, int E, int pm) {
  int lo = 0, hi = E;  // largest g with gtp[g] <= pm; empty groups are skipped
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (gtp[mid] <= pm) lo = mid; else hi = mid;
  }
  return lo;
}

// ============================================================================
// Offline calibration of D
// ============================================================================
// The MACAQ page lists calibration among the offline steps without a rule; the
// rule here is the square-root range balance D[k] = clamp(sqrt(a / w), 1e-2,
// 1e2) per expert and input channel, a = max |x[:, k]| over the expert's
// calibration rows, w = max |W[:, k]| over its weight rows, in binary64 and
// rounded once to fp32 (w = 0 < a gives 1e2, a = w = 0 gives 1, an expert with
// no rows gives 1).  A cluster of kCalibCluster CTAs per (64 channels, expert)
// splits the weight rows and the calibration rows; in each CTA 1024 threads =
// 64 channels x 16 row lanes, whose maxima are combined in shared memory; rank 0
// then combines the CTAs' maxima through distributed shared memory.  64 channels
// keep each warp's loads on whole 128-byte (W) and 64-byte (x) row segments
// while giving K / 8 CTAs per expert (128 for K = 1024), enough to cover the SMs.
constexpr int kCalibCluster = 8;
constexpr int kCalibCols = 64;
constexpr int kCalibLanes = 1024 / kCalibCols;
struct CalibParams {
  const uint16_t* x;  // bf16 [T, K]
  const float* W;     // [E, N, K]
  const int64_t* gl;  // group_list (validated by the host) or nullptr: every row is expert 0's
  int type;
  int E, N, K;
  int64_t T;
  float* D;           // [E, K]
};

__global__ void __launch_bounds__(1024) calibrate_kernel(const __grid_constant__ CalibParams p) {
  __shared__ float sa[kCalibLanes][kCalibCols], sw[kCalibLanes][kCalibCols];
  const int c = threadIdx.x % kCalibCols, lanes = threadIdx.x / kCalibCols;
  const int rank = static_cast<int>(cluster_ctarank());
  const int e = blockIdx.y;
  const int64_t k = static_cast<int64_t>(blockIdx.x / kCalibCluster) * kCalibCols + c;
  // this thread's rows: lane + kCalibLanes rank, then every kCalibLanes x kCalibCluster
  const int first = lanes + kCalibLanes * rank, stride = kCalibLanes * kCalibCluster;
  float w = 0.f, a = 0.f;  // maxima of magnitudes: exact in any order
  {
    // eight independent loads in flight per thread (one at a time would wait a
    // full memory latency per row)
    float wm[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    const float* wp = p.W + static_cast<int64_t>(e) * p.N * p.K + k;
    int n = first;
    for (; n + 7 * stride < p.N; n += 8 * stride) {
#pragma unroll
      for (int u = 0; u < 8; ++u) wm[u] = fmaxf(wm[u], fabsf(__ldg(wp + static_cast<int64_t>(n + u * stride) * p.K)));
    }
    for (; n < p.N; n += stride) wm[0] = fmaxf(wm[0], fabsf(__ldg(wp + static_cast<int64_t>(n) * p.K)));
#pragma unroll
    for (int u = 0; u < 8; ++u) w = fmaxf(w, wm[u]);
  }
  int64_t rows = 0;
  auto scan = [&](int64_t r0, int64_t r1) {
    float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int64_t r = r0 + first;
    for (; r + 7 * stride < r1; r += 8 * stride) {
#pragma unroll
      for (int u = 0; u < 8; ++u) am[u] = fmaxf(am[u], fabsf(bf16lo(__ldg(p.x + (r + u * stride) * p.K + k))));
    }
    for (; r < r1; r += stride) am[0] = fmaxf(am[0], fabsf(bf16lo(__ldg(p.x + r * p.K + k))));
#pragma unroll
    for (int u = 0; u < 8; ++u) a = fmaxf(a, am[u]);
  };
  if (p.gl == nullptr) {
    scan(0, p.T);
    rows = p.T;
  } else {
    int64_t r0 = 0;
    for (int j = 0; j < p.E; ++j) {  // list entry j: its rows and the expert they use
      int64_t cnt;
      int ex = j;
      if (p.type == 2) {
        ex = static_cast<int>(p.gl[2 * j]);
        cnt = p.gl[2 * j + 1];
      } else {
        cnt = p.type == 1 ? p.gl[j] : p.gl[j] - (j > 0 ? p.gl[j - 1] : 0);
      }
      if (ex == e) {
        scan(r0, r0 + cnt);
        rows += cnt;
      }
      r0 += cnt;
    }
  }
  sa[lanes][c] = a;
  sw[lanes][c] = w;
  __syncthreads();
  if (lanes == 0) {  // this CTA's maxima into row 0
    for (int l = 1; l < kCalibLanes; ++l) {
      sa[0][c] = fmaxf(sa[0][c], sa[l][c]);
      sw[0][c] = fmaxf(sw[0][c], sw[l][c]);
    }
  }
  cluster_sync_all();  // every CTA's maxima are in its shared memory
  if (rank == 0 && lanes == 0) {
    a = 0.f;
    w = 0.f;
    for (int o = 0; o < kCalibCluster; ++o) {
      a = fmaxf(a, ld_dsmem_f32(mapa_shared(smem_u32(&sa[0][c]), static_cast<uint32_t>(o))));
      w = fmaxf(w, ld_dsmem_f32(mapa_shared(smem_u32(&sw[0][c]), static_cast<uint32_t>(o))));
    }
    double d;
    if (rows == 0 || (a == 0.f && w == 0.f)) d = 1.0;
    else if (w == 0.f) d = 1e2;
    else d = sqrt(static_cast<double>(a) / static_cast<double>(w));  // IEEE divide and square root
    d = fmin(fmax(d, 1e-2), 1e2);
    p.D[static_cast<int64_t>(e) * p.K + k] = static_cast<float>(d);
  }
  cluster_sync_all();  // no CTA leaves while rank 0 may still read its shared memory
}

// ============================================================================
// Quantise-once: activation prologue over every row into tile images
// ============================================================================
// Work unit = one 32-row slab of a 128-row tile x one K tile: thread (tr, c) =
// (threadIdx.x / 8, threadIdx.x % 8) takes row tr of the slab and its 32-element
// block c.  Only slabs that hold rows are enumerated: dense, slab s is rows
// [32 s, 32 s + 32) of x (quarter s % 4 of tile s / 4); grouped, the slab table
// written by group_tables_kernel gives each slab's expert, first row of x, row
// count and quarter.  Rows past a slab's end are neither read nor written: the
// GEMM never stores the output rows they feed (a row of the product depends on
// its own activation row only).  Unit u is slab u % L of K tile u / L; the grid
// is persistent, each CTA stepping through units blockIdx.x, + gridDim.x, ...
// with the slab and K tile advanced incrementally (no division per unit).
// Every thread keeps the activations of its next kQuantAhead units in flight
// with cp.async into its own slots of a shared-memory ring (no registers held),
// so HBM streams while the ALUs work.
struct QuantParams {
  const uint16_t* x;
  const float* D;       // [E, K]
  uint8_t* Aq;          // [tiles][KT] activation images of kActImageBytes
  int M, K;
  const int4* slabs;    // grouped: slab table (nullptr: dense)
  const int* nslabs;    // grouped: its length
  const int* valid;
  int plain;            // plain MXFP4 (no D, no Hadamard; D not read)
};

// Quantise-once prologue over all rows.  A CTA owns one K tile and a contiguous
// run of 32-row slabs (dense: rows 32 s..; grouped: the slab table, in group
// order, copied into shared memory up front so that no global read sits on the
// path to the next copy); a thread owns row tr of the slab and the 32-channel
// block c of the K tile, i.e. one MX block per slab.  Each thread streams its
// rows kQuantDepth - 1 slabs ahead through a ring in shared memory (cp.async,
// chunk-major: a warp's 16-byte loads of chunk j are 512 consecutive bytes) and
// reads back only what it copied itself, so the ring needs no barrier.  The
// block's 32 reciprocals stay in registers while consecutive slabs use the same
// row of D (dense: always; grouped: until the group changes, a CTA-uniform
// event); the D values of a grouped slab travel in the ring with its
// activations, so a change of group costs no global round trip.
constexpr int kQuantCtasPerSm = 2;
constexpr int kQuantDepth = 4;             // ring slots: the slab being encoded and three ahead
constexpr int kQuantSlotBytes = 256 * 64;  // one slab: 256 threads x one 32-element block
constexpr int kQuantDOff = kQuantDepth * kQuantSlotBytes;          // then [kQuantDepth][256] D values
constexpr int kQuantSmem = kQuantDOff + kQuantDepth * 256 * 4;
constexpr int kQuantTab = 256;             // slab-table entries a CTA keeps in shared memory

__global__ void __launch_bounds__(256, kQuantCtasPerSm) quant_tiles_kernel(const __grid_constant__ QuantParams p) {
  extern __shared__ __align__(16) uint8_t qsmem[];  // ring [kQuantDepth][4 chunks][256 threads][16], then D
  float* dring = reinterpret_cast<float*>(qsmem + kQuantDOff);
  __shared__ __align__(16) float rs[kQRcpTile];
  __shared__ int4 tab[kQuantTab];
  pdl_trigger();  // the GEMM may start streaming weights; it waits for our results before reading them
  pdl_wait();     // x (and the grouped tables) may come from the preceding kernels
  const int KT = p.K / kKTile;
  const bool grouped = p.slabs != nullptr;
  int L = (p.M + 31) / 32;
  if (grouped) {
    if (*p.valid == 0) return;
    L = *p.nslabs;
  }
  // the grid is KT x per_kt CTAs: CTA (kt, j) takes slabs [j q, (j + 1) q)
  const int per_kt = static_cast<int>(gridDim.x) / KT;
  const int kt = static_cast<int>(blockIdx.x) % KT, j = static_cast<int>(blockIdx.x) / KT;
  const int q = (L + per_kt - 1) / per_kt;
  const int s0 = j * q;
  const int n = min(L, s0 + q) - s0;  // slabs of this CTA
  if (L <= 0 || j >= per_kt || n <= 0) return;
  if (grouped) {
    for (int i = threadIdx.x; i < min(n, kQuantTab); i += blockDim.x) tab[i] = p.slabs[s0 + i];
    __syncthreads();
  }
  // slab i of the run: (group, first row, rows, quarter = 32-row slot in the tile images)
  auto slab = [&](int i) -> int4 {
    if (grouped) return i < kQuantTab ? tab[i] : p.slabs[s0 + i];
    const int sl = s0 + i;
    return make_int4(0, sl * 32, min(32, p.M - sl * 32), sl);
  };
  const int tr = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int64_t k0 = static_cast<int64_t>(kt) * kKTile;
  // copies this thread's 64 bytes of slab i (grouped: and the D value of channel
  // k0 + threadIdx.x of its group) into ring slot `slot`; one group per slab
  auto fetch = [&](int i, int slot) {
    if (i < n) {
      const int4 e = slab(i);
      if (grouped && !p.plain)
        cp_async4(dring + slot * 256 + threadIdx.x, p.D + static_cast<int64_t>(e.x) * p.K + k0 + threadIdx.x);
      if (tr < e.z) {
        const uint16_t* src = p.x + (static_cast<int64_t>(e.y) + tr) * p.K + k0 + c * kBlk;
        uint8_t* dst = qsmem + slot * kQuantSlotBytes + threadIdx.x * 16;
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) cp_async16(dst + 4096 * ii, src + 8 * ii);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int i = 0; i < kQuantDepth - 1; ++i) fetch(i, i);
  float2 r2[16];
  int group = -1;  // the D row whose reciprocals r2 holds
  int slot = 0;    // ring slot of slab i
  for (int i = 0; i < n; ++i) {
    fetch(i + kQuantDepth - 1, slot == 0 ? kQuantDepth - 1 : slot - 1);  // the slot slab i - 1 freed
    const int4 e = slab(i);
    cp_async_wait<kQuantDepth - 1>();  // this thread's copies of slab i have landed
    if (!p.plain && e.x != group) {
      __syncthreads();  // every thread holds the previous reciprocals in registers already
      const float d = grouped ? dring[slot * 256 + threadIdx.x] : __ldg(p.D + k0 + threadIdx.x);
      rs[qrcp_index(threadIdx.x)] = __frcp_rn(d);
      __syncthreads();
      load_rcp_block(rs + c * kQRcpStride, r2);
      group = e.x;
    }
    if (tr < e.z) {
      const uint4* xs = reinterpret_cast<const uint4*>(qsmem + slot * kQuantSlotBytes) + threadIdx.x;
      const uint4 xv[4] = {xs[0], xs[256], xs[512], xs[768]};
      uint4 cv;
      uint32_t sc;
      if (p.plain) act_block_plain(xv, cv, sc);
      else act_block(xv, r2, cv, sc);
      const int t = (e.w & 3) * 32 + tr;
      uint8_t* img = p.Aq + (static_cast<size_t>(e.w >> 2) * KT + kt) * kActImageBytes;
      *reinterpret_cast<uint4*>(img + code_chunk_offset(t, c)) = cv;
      img[kTileCodeBytes + sf_offset(t, c)] = static_cast<uint8_t>(sc);
    }
    if (++slot == kQuantDepth) slot = 0;
  }
  cp_async_wait<0>();  // no copy may still be writing this CTA's shared memory at exit
}

// ============================================================================
// Persistent GEMM over tile images
// ============================================================================
struct GemmParams {
  const uint8_t* Wq;  // weight images, pairs per K tile (weight_image)
  const uint8_t* Ws;
  const uint8_t* Aq;  // activation images [tiles][KT], kActImageBytes each
  uint16_t* y;        // bf16 [M, N]
  int M, N, K, NT, KT, E, MT;
  const int64_t* goff;  // grouped tables (nullptr: dense with MT tiles)
  const int* gtp;
  const int* gexp;      // expert of each group_list entry
  const int* valid;
  int32_t* status;
  int wait_for_producer;  // dense: 1 when launched as a programmatic dependent of the quantiser
  int NT2;                // 256-wide output tiles: ceil(NT / 2)
  int stages;             // pipeline depth (gemm::stages_for(E))
  float out_scale;        // 2^-5 (MACAQ: undoes the two unnormalised Hadamards), 1 (plain MXFP4)
  const float* bias;      // fp32 [E][N] (expert g's row for its tiles) or nullptr
  int act;                // act_type: 0 none, 1 RELU, 2 GELU_TANH, 4 FAST_GELU, 5 SILU
  const uint64_t* wq_list;  // weight-list form: [E] addresses of each expert's images (else nullptr)
  const uint64_t* ws_list;
  uint8_t* y8;              // FP8 output: E4M3 codes [M, N] written instead of y (else nullptr)
  float y8_scale;           // multiplies the epilogue value before the E4M3 rounding
};

// Epilogue of 32 accumulator columns of one thread's row, loaded into
// registers: v = acc * out_scale (+ bias[n]), then the activation, packed to 16
// BF16 pairs.  kEpi < 0: scaling only (no bias, no activation); otherwise
// act_type kEpi with an optional bias, read from the tile's bias staged in
// shared memory (sb: the 32 values of these columns; zero past N).
template <int kEpi>
__device__ __forceinline__ float2 epi_pair(const uint32_t (&r)[32], int e, float2 os2, const float* sb) {
  const float2 a = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
  if constexpr (kEpi < 0) {
    return fmul2(a, os2);
  } else {
    const float2 b = *reinterpret_cast<const float2*>(sb + 2 * e);  // warp-uniform: a broadcast
    return act_pair<kEpi>(ffma2(a, os2, b));
  }
}
template <int kEpi>
__device__ __forceinline__ void finish32(const uint32_t (&r)[32], float os, const float* sb, uint32_t* pk) {
  const float2 os2 = make_float2(os, os);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    const float2 y = epi_pair<kEpi>(r, e, os2, sb);
    pk[e] = pack_bf16x2(y.x, y.y);
  }
}
// The same 32 columns as FP8 E4M3 codes (8 words, column 0 in the lowest byte):
// each value times y8_scale in FP32, then rounded to nearest even with saturation
// at +-448 (cvt.rn.satfinite; NaN stays NaN).
__device__ __forceinline__ uint8_t e4m3_1(float v) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
  return static_cast<uint8_t>(r & 0xFFu);
}
__device__ __forceinline__ uint32_t e4m3x4(float2 a, float2 b) {
  uint16_t lo, hi;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(lo) : "f"(a.x), "f"(a.y));
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(hi) : "f"(b.x), "f"(b.y));
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}
template <int kEpi>
__device__ __forceinline__ void finish32_fp8(const uint32_t (&r)[32], float os, const float* sb, float y8s,
                                             uint32_t* pk) {
  const float2 os2 = make_float2(os, os), s2 = make_float2(y8s, y8s);
#pragma unroll
  for (int e = 0; e < 16; e += 2) {
    const float2 y0 = fmul2(epi_pair<kEpi>(r, e, os2, sb), s2);
    const float2 y1 = fmul2(epi_pair<kEpi>(r, e + 1, os2, sb), s2);
    pk[e / 2] = e4m3x4(y0, y1);
  }
}

// Large M: the MMA is not swapped.  Operand A = a 128-token activation tile,
// operand B = 256 output channels of weights (two 128-row weight images side by
// side in shared memory), D[t][n] in TMEM with one token per lane, so each
// epilogue thread owns a contiguous run of an output row.  An M = 128 MMA takes
// about as long to issue at N = 128 as at N = 256, so the wider tile doubles the
// work per instruction.
namespace gemm {
constexpr int kMaxStages = 4;
constexpr int kThreads = 352;  // warp 0 producer, warp 1 MMA, warps 2-9 epilogue, warp 10 scale copies
constexpr int kTileN = 256;
// A stage takes three copies: the weight codes of an image pair (32 KB), the
// activation image (codes then scales, 17 KB) and the pair's scales (2 KB).
constexpr int kOffB = 0;                                    // weight codes, 256 rows (two images)
constexpr int kOffA = 2 * kTileCodeBytes;                   // activation codes, 128 rows
constexpr int kOffSfa = kOffA + kTileCodeBytes;             // activation scales (same copy)
constexpr int kOffSfb = kOffSfa + kTileSfBytes;             // weight scales of the two images
constexpr int kStageBytes = kOffSfb + 2 * kTileSfBytes;     // 52224
constexpr int kStagingBytes = kRowsTile * 64 * 2;           // 128 rows x 64 columns of BF16, swizzled
constexpr int kBiasBytes = kTileN * 4;                       // the tile's 256 bias values
constexpr int kFixedBytes = kStagingBytes + 256 + kBiasBytes;  // staging, barriers and flags, bias
// TMEM: the accumulator in columns 0-255; from column 256, 24 columns of scales per
// stage (activation scales 8, weight scales 16)
constexpr int kTmemCols = 512;
constexpr int kSfCol = 256;
constexpr int kSfCols = 24;
static_assert(kSfCol + kSfCols * kMaxStages <= kTmemCols, "scale slots fit the allocation");
static_assert(kStageBytes % 1024 == 0, "stage alignment");
constexpr size_t kSmemLimit = 227 * 1024;
// goff (8), gtp (4), gexp (4) per entry; the weight-list form adds the two image
// address tables (8 + 8 per expert)
__host__ __device__ constexpr size_t group_bytes(int E, bool list = false) {
  return E > 0 ? static_cast<size_t>(E + 1) * 16 + 16 + (list ? static_cast<size_t>(E) * 16 : 0) : 0;
}
// four stages when the group tables leave room for them, else three
__host__ __device__ constexpr int stages_for(int E, bool list = false) {
  return 1024 + static_cast<size_t>(kMaxStages) * kStageBytes + kFixedBytes + group_bytes(E, list) <= kSmemLimit
             ? kMaxStages
             : kMaxStages - 1;
}
__host__ __device__ constexpr size_t smem_bytes(int E, bool list = false) {
  return 1024 + static_cast<size_t>(stages_for(E, list)) * kStageBytes + kFixedBytes + group_bytes(E, list);
}
static_assert(smem_bytes(0) <= kSmemLimit && smem_bytes(1024, true) <= kSmemLimit, "shared memory");
}  // namespace gemm

struct GemmTile {
  int g, m0, rows, pm, nt;  // nt: the first of the tile's two weight images
};

__device__ __forceinline__ GemmTile gemm_tile(const GemmParams& p, int idx, int mtiles, const int64_t* goff,
                                              const int* gtp, const int* gexp) {
  GemmTile t;
  t.pm = idx % mtiles;
  t.nt = 2 * (idx / mtiles);
  if (gtp == nullptr) {
    t.g = 0;
    t.m0 = t.pm * kRowsTile;
    t.rows = min(kRowsTile, p.M - t.m0);
  } else {
    const int e = find_group(gtp, p.E, t.pm);  // list entry; its rows use expert gexp[e]
    t.g = gexp[e];
    t.m0 = static_cast<int>(goff[e]) + (t.pm - gtp[e]) * kRowsTile;
    t.rows = min(kRowsTile, static_cast<int>(goff[e + 1]) - t.m0);
  }
  return t;
}

// Scale copies of one 256-K stage of the wide tile into its TMEM slot.  Weight
// scales: for each group of four scale blocks, eight columns (rows 0-127 of B, then
// rows 128-255); activation scales four columns.
//
// The copies are issued by a warp of their own, not by the MMA issuer: measured on
// B200, a thread whose instruction stream mixes tcgen05.cp with an mbarrier wait
// between stages issues block-scaled MMAs at ~190-200 cycles each instead of ~140,
// while an issuer that only waits and issues MMAs keeps ~148.
__device__ __forceinline__ void scale_copies_wide(uint64_t sfadesc, uint64_t sfbdesc, uint32_t sf_col) {
  constexpr uint64_t kBlk512 = 512 >> 4, kImg = kTileSfBytes >> 4;
  tc_cp_32x128b_warpx4(sf_col, sfadesc);
  tc_cp_32x128b_warpx4(sf_col + 4, sfadesc + kBlk512);
  tc_cp_32x128b_warpx4(sf_col + 8, sfbdesc);
  tc_cp_32x128b_warpx4(sf_col + 12, sfbdesc + kImg);
  tc_cp_32x128b_warpx4(sf_col + 16, sfbdesc + kBlk512);
  tc_cp_32x128b_warpx4(sf_col + 20, sfbdesc + kImg + kBlk512);
}

// The four MMAs of one 256-K stage of the wide tile: D (+)= A x B^T with N = 256,
// scales from the stage's TMEM slot (scale_copies_wide).
__device__ __forceinline__ void mma_stage_wide(uint64_t adesc, uint64_t bdesc, uint32_t sf_col, uint32_t d_tmem,
                                               uint32_t idesc_lo, uint32_t idesc_hi, bool first) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t sfid = static_cast<uint32_t>(k & 1) * 2u;
    const uint32_t sfa = (sf_col + (k >> 1) * 4) | (sfid << 30);
    const uint32_t sfb = (sf_col + 8 + (k >> 1) * 8) | (sfid << 30);
    tc_mma_mxf4(d_tmem, adesc + 2 * k, bdesc + 2 * k, (k & 1) ? idesc_hi : idesc_lo, sfa, sfb,
                (!first || k > 0) ? 1u : 0u);
  }
}

// Scale copies of one 256-K stage: sfadesc / sfbdesc describe the stage's scale
// images (two 512-byte blocks each).  A descriptor's start address field counts
// 16-byte units, so the descriptor of a later address is the first one plus the
// distance / 16.  Issued by a warp other than the MMA issuer (see scale_copies_wide).
__device__ __forceinline__ void scale_copies(uint64_t sfadesc, uint64_t sfbdesc, uint32_t sfa_col, uint32_t sfb_col) {
  tc_cp_32x128b_warpx4(sfa_col, sfadesc);
  tc_cp_32x128b_warpx4(sfa_col + 4, sfadesc + (512 >> 4));
  tc_cp_32x128b_warpx4(sfb_col, sfbdesc);
  tc_cp_32x128b_warpx4(sfb_col + 4, sfbdesc + (512 >> 4));
}

// The four MMAs of one 256-K stage: D (+)= A-tile x B-tile^T; adesc / bdesc describe
// the stage's code images, the scales sit in TMEM from sfa_col / sfb_col.
__device__ __forceinline__ void mma_stage(uint64_t adesc, uint64_t bdesc, uint32_t sfa_col, uint32_t sfb_col,
                                          uint32_t d_tmem, uint32_t idesc_lo, uint32_t idesc_hi, bool first) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    // scale bytes 0-1 of each 32-bit TMEM word for the first 64 K, bytes 2-3 for the next;
    // each 64-K step is 32 bytes further along the code rows
    const uint32_t sfid = static_cast<uint32_t>(k & 1) * 2u;
    const uint32_t sfa = (sfa_col + (k >> 1) * 4) | (sfid << 30);
    const uint32_t sfb = (sfb_col + (k >> 1) * 4) | (sfid << 30);
    tc_mma_mxf4(d_tmem, adesc + 2 * k, bdesc + 2 * k, (k & 1) ? idesc_hi : idesc_lo, sfa, sfb,
                (!first || k > 0) ? 1u : 0u);
  }
}

// kEpi < 0: the output is the scaled sum; kEpi = act_type (0, 1, 2, 4, 5): an
// optional bias (p.bias) and that activation are applied in the epilogue.
template <int kEpi>
__global__ void __launch_bounds__(gemm::kThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using namespace gemm;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint8_t* staging = smem + S * kStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(staging + kStagingBytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* sfull = empty + kMaxStages;  // the stage's scales are in TMEM
  uint64_t* accf = sfull + kMaxStages;   // accumulator complete
  uint64_t* acce = accf + 1;             // accumulator drained by the epilogue
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_flag = abort_flag + 1;
  int64_t* goff = nullptr;
  int* gtp = nullptr;
  int* gexp = nullptr;
  uint64_t* wql = nullptr;  // weight-list form: each expert's code / scale image addresses
  uint64_t* wsl = nullptr;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int mtiles = p.MT;
  if (p.gtp != nullptr) {
    pdl_wait();  // tables and activation images come from the preceding kernels
    if (*p.valid == 0) return;
    goff = reinterpret_cast<int64_t*>(reinterpret_cast<uint8_t*>(full) + 256 + kBiasBytes);
    gtp = reinterpret_cast<int*>(goff + p.E + 1);
    gexp = gtp + p.E + 1;
    if (p.wq_list != nullptr) {
      wql = reinterpret_cast<uint64_t*>(goff + 2 * (p.E + 1));  // after goff, gtp, gexp (16 bytes per entry + 16)
      wsl = wql + p.E;
    }
    for (int i = threadIdx.x; i <= p.E; i += blockDim.x) {
      goff[i] = p.goff[i];
      gtp[i] = p.gtp[i];
      if (i < p.E) gexp[i] = p.gexp[i];
      if (wql != nullptr && i < p.E) {
        wql[i] = p.wq_list[i];
        wsl[i] = p.ws_list[i];
      }
    }
    __syncthreads();
    mtiles = gtp[p.E];
  }
  const int total = mtiles * p.NT2;
  if (static_cast<int>(blockIdx.x) >= total) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sfull[s], 1);
    }
    mbar_init(accf, 1);
    mbar_init(acce, 8);  // one arrival per epilogue warp
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int my_tiles = (total - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                       static_cast<int>(gridDim.x);
  const int KT = p.KT;

  if (warp == 0) {
    // ================= producer: bulk copies of weight and activation images =================
    // A bulk-copy instruction holds up the path that issued it until the engine has
    // taken its copy in, so the three copies of a stage are not issued one after
    // another: the warp stays converged and one predicated instruction starts them
    // together.  A single warp has no other work to hide its own latency behind, so
    // the source of each copy is stepped along, not recomputed, and worked out
    // before the wait.
    const int slots = my_tiles * KT;
    const int pre = min(S, slots);
    // Copy c of a stage: 0 activation image, 1 codes of the weight pair, 2 its
    // scales.  Gives k tile 0 of this CTA's i-th output tile; k tile kt is
    // kt * step further on.
    auto source = [&](int i, int c, const uint8_t*& src, uint32_t& bytes, uint32_t& doff, uint32_t& step) {
      const GemmTile t = gemm_tile(p, blockIdx.x + i * gridDim.x, mtiles, goff, gtp, gexp);
      // stacked weights: expert t.g's images follow the others'; weight list: its own base
      const size_t img = weight_image(wql != nullptr ? 0 : t.g, t.nt, 0, p.NT2, KT);
      const uint8_t* wq = wql != nullptr ? reinterpret_cast<const uint8_t*>(wql[t.g]) : p.Wq;
      const uint8_t* ws = wql != nullptr ? reinterpret_cast<const uint8_t*>(wsl[t.g]) : p.Ws;
      bytes = c == 0 ? kActImageBytes : c == 1 ? 2 * kTileCodeBytes : 2 * kTileSfBytes;
      step = c == 0 ? kActImageBytes : bytes;
      src = c == 0 ? p.Aq + static_cast<size_t>(t.pm) * KT * kActImageBytes
                   : (c == 1 ? wq + img * kTileCodeBytes : ws + img * kTileSfBytes);
      doff = c == 0 ? kOffA : c == 1 ? kOffB : kOffSfb;
    };
    const uint8_t* src;
    uint32_t bytes, doff, step;
    if (lane == 0)
      for (int j = 0; j < pre; ++j) mbar_arrive_expect_tx(&full[j], kStageBytes);
    __syncwarp();
    {  // first stages: weights (lane 2s + w: copy 1 + w of stage s) before the quantiser's wait
      const int j = min(lane >> 1, pre - 1);
      source(j / KT, 1 + (lane & 1), src, bytes, doff, step);
      bulk_g2s_if(lane < 2 * pre, smem + j * kStageBytes + doff, src + (j % KT) * step, bytes, &full[j]);
    }
    if (p.wait_for_producer) pdl_wait();
    {  // then their activations (lane s: copy 0 of stage s)
      const int j = min(lane, pre - 1);
      source(j / KT, 0, src, bytes, doff, step);
      bulk_g2s_if(lane < pre, smem + j * kStageBytes + doff, src + (j % KT) * step, bytes, &full[j]);
    }
    // from then on lane c < 3 streams copy c of every stage
    const int c = lane < 3 ? lane : 0;
    int kt = pre % KT, i = pre / KT, stage = 0;
    uint32_t phase = 1;  // slots from `pre` on reuse stages released once before
    if (pre < slots) source(i, c, src, bytes, doff, step);
    for (int j = pre; j < slots; ++j) {
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitTimeoutNs) ? 1 : 0;
        if (ok) mbar_arrive_expect_tx(&full[stage], kStageBytes);
      }
      __syncwarp();  // the stage is free for every lane, not only the one that waited
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      bulk_g2s_if(lane < 3, smem + stage * kStageBytes + doff, src + kt * step, bytes, &full[stage]);
      if (++stage == S) {
        stage = 0;
        phase ^= 1;
      }
      if (++kt == KT) {
        kt = 0;
        if (j + 1 < slots) source(++i, c, src, bytes, doff, step);
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      const uint32_t idesc_lo = idesc_mxf4(128, kTileN, 0, 0);
      const uint32_t idesc_hi = idesc_mxf4(128, kTileN, 2, 2);
      const uint64_t code0 = sdesc_kmajor_sw128(smem_u32(smem));
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < my_tiles && ok; ++i) {
        if (!mbar_wait(acce, (i & 1) ^ 1, abort_flag, kWaitTimeoutNs)) break;
        tc_fence_after();
        for (int kt = 0; kt < KT; ++kt) {
          // operands in shared memory, then their scales in TMEM (warp 10)
          if (!mbar_wait(&full[stage], phase, abort_flag, kWaitTimeoutNs) ||
              !mbar_wait(&sfull[stage], phase, abort_flag, kWaitTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t so = static_cast<uint32_t>(stage * kStageBytes) >> 4;
          mma_stage_wide(code0 + so + (kOffA >> 4), code0 + so + (kOffB >> 4), tmem + kSfCol + kSfCols * stage, tmem,
                         idesc_lo, idesc_hi, kt == 0);
          tc_commit(&empty[stage]);
          if (++stage == S) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        tc_commit(accf);
      }
    }
  } else if (warp == 10) {
    // ================= scale copies: each stage's scales into its TMEM slot =================
    // A slot is rewritten only after its stage was refilled, which the producer does
    // only after the MMAs that read the slot's previous contents completed.
    if (lane == 0) {
      const uint64_t sf0 = sdesc_sf_block(smem_u32(smem));
      const int slots = my_tiles * KT;
      int stage = 0;
      uint32_t phase = 0;
      for (int j = 0; j < slots; ++j) {
        if (!mbar_wait(&full[stage], phase, abort_flag, kWaitTimeoutNs)) break;
        const uint32_t so = static_cast<uint32_t>(stage * kStageBytes) >> 4;
        scale_copies_wide(sf0 + so + (kOffSfa >> 4), sf0 + so + (kOffSfb >> 4), tmem + kSfCol + kSfCols * stage);
        tc_commit(&sfull[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else {
    // ================= epilogue: TMEM -> x 2^-5 -> BF16 -> staged chunks -> coalesced rows =================
    // Warp w reads TMEM lanes 32 (w % 4) .. + 31 (accumulator rows) and columns
    // 128 h .. + 127 with h = (w - 2) / 4.  Rows go out in 64-column chunks staged
    // in shared memory with their 16-byte pieces XOR-swizzled by the row
    // (conflict-free writes and reads).
    const int q = warp & 3, h = (warp - 2) >> 2;
    const int et = threadIdx.x - 64;
    const float os = p.out_scale;
    const int tl = q * 32 + lane;
    float* sbias = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 256);  // [256]
    for (int i = 0; i < my_tiles; ++i) {
      const GemmTile t = gemm_tile(p, blockIdx.x + i * gridDim.x, mtiles, goff, gtp, gexp);
      if constexpr (kEpi >= 0) {
        // the tile's 256 bias values, one per thread: every later read is a shared-memory
        // broadcast instead of a global load in the middle of the epilogue's dependency chain
        const int n = t.nt * kRowsTile + et;
        sbias[et] = (p.bias != nullptr && n < p.N) ? __ldg(p.bias + static_cast<int64_t>(t.g) * p.N + n) : 0.f;
      }
      if (et == 0) *epi_flag = mbar_wait(accf, i & 1, abort_flag, kWaitTimeoutNs) ? 1 : 0;
      named_bar_sync(1, 256);  // also: every thread has finished reading the previous tile's staging and bias
      if (!*epi_flag) break;
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + h * 128;
      // Chunk ch of the tile = columns 64 ch .. + 63, held by half ch / 2.  A chunk is
      // staged with its 16-byte pieces XOR-swizzled by the row, then all 256
      // threads store it as coalesced 128-byte row runs.
      const int c = et & 7;  // 16-byte piece of a 128-byte row run
      auto stage_chunk = [&](const uint32_t* src) {
        uint8_t* srow = staging + tl * 128;
#pragma unroll
        for (int g = 0; g < 8; ++g)
          *reinterpret_cast<uint4*>(srow + ((g ^ (tl & 7)) << 4)) =
              make_uint4(src[4 * g], src[4 * g + 1], src[4 * g + 2], src[4 * g + 3]);
      };
      auto store_chunk = [&](int ch) {
        const int n0 = t.nt * kRowsTile + ch * 64;
        if (n0 + 8 * c < p.N) {
#pragma unroll 4
          for (int rr = et >> 3; rr < t.rows; rr += 32) {
            const uint4 o = *reinterpret_cast<const uint4*>(staging + rr * 128 + ((c ^ (rr & 7)) << 4));
            *reinterpret_cast<uint4*>(p.y + static_cast<int64_t>(t.m0 + rr) * p.N + n0 + 8 * c) = o;
          }
        }
      };
      // The row's 128 accumulator columns are loaded into registers with one wait
      // and the accumulator is handed back at once: the next tile's MMAs overlap
      // the scaling, bias and activation (bias from shared memory) and the write-out.
      uint32_t r[4][32];
#pragma unroll
      for (int j = 0; j < 4; ++j) tmem_ld_32x32b_x32(taddr + 32 * j, r[j]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce);
      uint32_t pk[64];
      if (p.y8 == nullptr) {
#pragma unroll
        for (int j = 0; j < 4; ++j) finish32<kEpi>(r[j], os, sbias + h * 128 + 32 * j, pk + 16 * j);
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if ((ch >> 1) == h) stage_chunk(pk + (ch & 1) * 32);
          named_bar_sync(1, 256);
          store_chunk(ch);
          if (ch < 3) named_bar_sync(1, 256);  // read out before the next chunk overwrites it
        }
      } else {
        // FP8 output: a half's 128 columns are 128 bytes of a row, one staged chunk
        // per half (the same swizzled staging), stored as 16-column pieces
#pragma unroll
        for (int j = 0; j < 4; ++j) finish32_fp8<kEpi>(r[j], os, sbias + h * 128 + 32 * j, p.y8_scale, pk + 8 * j);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          if (ch == h) stage_chunk(pk);
          named_bar_sync(1, 256);
          const int n0 = t.nt * kRowsTile + ch * 128;
          if (n0 + 16 * c < p.N) {
#pragma unroll 4
            for (int rr = et >> 3; rr < t.rows; rr += 32) {
              const uint4 o = *reinterpret_cast<const uint4*>(staging + rr * 128 + ((c ^ (rr & 7)) << 4));
              *reinterpret_cast<uint4*>(p.y8 + static_cast<int64_t>(t.m0 + rr) * p.N + n0 + 16 * c) = o;
            }
          }
          if (ch < 1) named_bar_sync(1, 256);
        }
      }
    }
  }

  if (*abort_flag && threadIdx.x == 0 && p.status) *p.status = MACAQ_ERR_DEVICE_TIMEOUT;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ============================================================================
// Small M: fused prologue + cluster split-K
// ============================================================================
struct FusedParams {
  const uint8_t* Wq;
  const uint8_t* Ws;
  const uint16_t* x;  // bf16 [M, K]
  const float* D;     // [K]
  uint16_t* y;
  int M, N, K, NT, KT, S;  // S = CTAs per cluster = K splits
  int32_t* status;
  int plain;               // plain MXFP4 (no D, no Hadamard; D not read)
  float out_scale;         // 2^-5 (MACAQ) or 1 (plain)
  const float* bias;       // fp32 [N] or nullptr
  int act;                 // act_type (act_value)
  uint8_t* dump_codes;     // test instantiation only: canonical [M, K/2] codes of the operand tiles
  uint8_t* dump_scales;    // and [M, K/32] scales, copied out of shared memory before each MMA
  uint8_t* y8;             // FP8 (E4M3) output instead of y (nullptr: BF16 into y)
  float y8_scale;
};

namespace fused {
constexpr int kStages = 4;
constexpr int kProWarps = 8;
// warp 0 producer, 1 MMA, 2-5 epilogue (warp 2 also issues the scale copies during
// the mainloop), 6-13 prologue
constexpr int kThreads = (6 + kProWarps) * 32;
template <int BT>
struct Cfg {
  static constexpr int kBBytes = BT * 128;
  static constexpr int kStageBytes = kTileCodeBytes + kBBytes + 2 * kTileSfBytes;
  static constexpr int kOffB = kTileCodeBytes;
  static constexpr int kOffSfa = kTileCodeBytes + kBBytes;
  static constexpr int kOffSfb = kOffSfa + kTileSfBytes;
  // receive buffer of the cluster reduction: slot [source rank][owned row][128] FP32;
  // S ranks own ceil(BT/S) rows each, so at most BT + 7 rows of slots
  static constexpr int kRecvOff = kStages * kStageBytes;
  static constexpr int kRecvBytes = (BT + 8) * kRowsTile * 4;
  static constexpr int kBarOff = kRecvOff + kRecvBytes;
  // The prologue warps work as kGroups groups, group g on the CTA's K tiles g,
  // g + kGroups, ...: a small token tile then has several K tiles in flight.
  static constexpr int kGroups = BT <= 16 ? 2 : 1;
  static constexpr int kGroupThreads = kProWarps * 32 / kGroups;
  static constexpr int kRbufOff = kBarOff + 256;  // per group, two K tiles of reciprocals
  static constexpr int kSmemBytes = 1024 + kRbufOff + kGroups * 2 * kQRcpTile * 4;
  // scale factors from kSfCol, 16 columns per stage
  static constexpr int kSfCol = BT < 32 ? 32 : BT;
  static constexpr int kTmemCols = kSfCol + 16 * kStages <= 64 ? 64 : kSfCol + 16 * kStages <= 128 ? 128 : 256;
  // 32-element blocks per prologue thread and per K tile
  static constexpr int kTasks = BT * 8 / kGroupThreads;
  static_assert(BT * 8 % kGroupThreads == 0, "whole blocks per thread");
  // reciprocals 1/D of a K tile per prologue thread
  static constexpr int kRcp = kKTile / kGroupThreads;
  static_assert(kKTile % kGroupThreads == 0, "whole reciprocals per thread");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};
}  // namespace fused

// Test instantiations: the activation operand tile of one K tile (BT rows of
// swizzled codes and its scale image) as the tensor core will read it, copied to
// canonical codes [M, K/2] and scales [M, K/32] by the MMA issuer between the
// wait for the tile and the MMAs that read it.  Only the CTAs of the first
// channel tile copy, so every (row, K tile) is written once.
template <int BT>
__device__ __forceinline__ void dump_act_tile(const uint8_t* bcode, const uint8_t* bsf, const FusedParams& p, int m0,
                                              int rows, int kt) {
  for (int t = 0; t < rows; ++t) {
    const int64_t row = m0 + t;
    for (int c = 0; c < 8; ++c) {
      *reinterpret_cast<uint4*>(p.dump_codes + row * (p.K / 2) + kt * (kKTile / 2) + c * (kBlk / 2)) =
          *reinterpret_cast<const uint4*>(bcode + code_chunk_offset(t, c));
      p.dump_scales[row * (p.K / kBlk) + kt * (kKTile / kBlk) + c] = bsf[sf_offset(t, c)];
    }
  }
}

// kEpilogue: the bias / activation epilogue (p.bias, p.act) is compiled in.
// kDump: test instantiation copying the activation operand tiles out (dump_act_tile).
template <int BT, bool kEpilogue = false, bool kDump = false>
__global__ void __launch_bounds__(fused::kThreads, 1) fused_small_kernel(const __grid_constant__ FusedParams p) {
  using C = fused::Cfg<BT>;
  using fused::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* recv_bar = accf + 1;  // completes when every rank's partial rows for this CTA have landed
  uint64_t* sfull = recv_bar + 1;  // [kStages] the stage's scales are in TMEM
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(sfull + kStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_flag = abort_flag + 1;
  volatile int* pro_flag = abort_flag + 2;  // [group][2]
  float* rbuf = reinterpret_cast<float*>(smem + C::kRbufOff);
  float* part = reinterpret_cast<float*>(smem);  // local FP32 partial tile [BT][128], after the mainloop

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work that needs no kernel parameter goes first: the first read of the
  // parameters stalls each SM for hundreds of cycles (measured ~900).
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + fused::kProWarps / C::kGroups);
      mbar_init(&empty[s], 1);
      mbar_init(&sfull[s], 1);
    }
    mbar_init(&accf[0], 1);
    *abort_flag = 0;
  }
  const uint32_t rank = cluster_ctarank();
  const int cid = blockIdx.x / p.S;
  const int nt = cid % p.NT, mt = cid / p.NT;
  const int m0 = mt * BT, rows = min(BT, p.M - m0);
  const int kt0 = static_cast<int>(rank) * p.KT / p.S, kt1 = (static_cast<int>(rank) + 1) * p.KT / p.S;
  // split-K ownership: rank o reduces and writes rows [o * rpr, o * rpr + rows_of(o)) of the tile
  const int rpr = (BT + p.S - 1) / p.S;
  auto rows_of = [&](int o) { return max(0, min(rpr, BT - o * rpr)); };
  const bool split = p.S > 1;  // launched as a cluster of S CTAs; S == 1 touches no cluster state

  if (threadIdx.x == 0) {
    if (split) {
      mbar_init(recv_bar, 1);
      mbar_arrive_expect_tx(recv_bar, static_cast<uint32_t>(p.S * rows_of(static_cast<int>(rank)) * kRowsTile * 4));
    }
    fence_mbar_init();
  }
  const int nst = kt1 - kt0;                   // K tiles of this CTA
  const int pre = nst < kStages ? nst : kStages;  // first-use stages: no wait for a free slot
  // The weights do not depend on any earlier kernel.  A bulk copy holds its
  // issuing warp ~150 cycles, so only stage 0's two copies go out before the
  // set-up barrier (which every warp waits for); the other first-use stages
  // follow right after it.  Lanes 2j and 2j + 1 copy stage j's codes and scales.
  auto first_copies = [&](int j0, int j1) {
    if (lane == 0)
      for (int j = j0; j < j1; ++j) mbar_arrive_expect_tx(&full[j], kTileCodeBytes + kTileSfBytes);
    __syncwarp();
    const int j = min(j0 + (lane >> 1), j1 - 1);
    const bool sf = lane & 1;
    const size_t wt = weight_image(0, nt, kt0 + j, (p.NT + 1) / 2, p.KT);
    uint8_t* sb = smem + j * C::kStageBytes;
    bulk_g2s_if(lane < 2 * (j1 - j0), sf ? sb + C::kOffSfa : sb,
                sf ? p.Ws + wt * kTileSfBytes : p.Wq + wt * kTileCodeBytes, sf ? kTileSfBytes : kTileCodeBytes,
                &full[j]);
  };
  if (warp == 0) {
    __syncwarp();  // lane 0 initialised the barriers
    first_copies(0, 1);
  }
  // Activation prologue set-up.  Each thread computes whole 32-element blocks (the
  // rotation and the block maximum stay in its registers: no exchange between
  // lanes); a K tile of the smallest token tile is one block per thread of its
  // group.  Rows past the tile's end are computed on zeros, which encode to zero
  // codes and a zero scale.  Group g of the prologue warps takes the CTA's K tiles
  // g, g + kGroups, ...; the activation loads of its first kAhead K tiles are
  // issued as soon as x may be read, so they land while the rest of the CTA sets up.
  constexpr int kGT = C::kGroupThreads, kG = C::kGroups;
  constexpr int kAhead = C::kTasks <= 1 ? 2 : 1;
  const int pt = static_cast<int>(threadIdx.x) - 6 * 32;
  const int grp = pt / kGT, gt = pt % kGT;
  auto load = [&](int kt, uint4 (&xv)[C::kTasks][4], float (&d)[C::kRcp]) {
#pragma unroll
    for (int u = 0; u < C::kTasks; ++u) {
      const int task = gt + u * kGT, t = task >> 3, c = task & 7;
#pragma unroll
      for (int i = 0; i < 4; ++i) xv[u][i] = make_uint4(0, 0, 0, 0);
      if (t < rows) {
        const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m0 + t) * p.K +
                                                          static_cast<int64_t>(kt) * kKTile + c * kBlk);
#pragma unroll
        for (int i = 0; i < 4; ++i) xv[u][i] = __ldg(src + i);
      }
    }
#pragma unroll
    for (int e = 0; e < C::kRcp; ++e) d[e] = p.plain ? 1.f : __ldg(p.D + static_cast<int64_t>(kt) * kKTile + gt + e * kGT);
  };
  const int gst = nst > grp ? (nst - grp + kG - 1) / kG : 0;  // this group's K tiles
  auto kt_of = [&](int jj) { return kt0 + grp + kG * jj; };
  uint4 xpre[kAhead][C::kTasks][4];
  float dpre[kAhead][C::kRcp];
  if (warp >= 6) {
    pdl_wait();  // x and D may come from the previous kernel on the stream
#pragma unroll
    for (int jj = 0; jj < kAhead; ++jj)
      if (jj < gst) load(kt_of(jj), xpre[jj], dpre[jj]);
  }
  // (scale rows >= BT of the activation scale image are copied to TMEM but never
  // read: the MMA's N extent is BT)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // The next kernel on the stream may start its own set-up now; everything this
  // kernel reads that an earlier kernel may have written (x, D) or writes (y)
  // is touched only after griddepcontrol.wait below.  The offline-prepared
  // weights are read before it.
  pdl_trigger();
  // Remote shared memory may only be touched once every CTA of the cluster runs
  // (and has initialised its receive barrier): arrive now, wait before the
  // first remote access.
  if (split) cluster_arrive_release();
  bool cluster_waited = false;

  if (warp == 0) {
    // ---- producer: weight images; lanes 0 and 1 start a stage's two copies with one
    // instruction of the converged warp ----
    if (pre > 1) first_copies(1, pre);
    for (int j = pre; j < nst; ++j) {
      const int kt = kt0 + j, stage = j % kStages;
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait(&empty[stage], ((j / kStages) & 1) ^ 1, abort_flag, kWaitTimeoutNs) ? 1 : 0;
        if (ok) mbar_arrive_expect_tx(&full[stage], kTileCodeBytes + kTileSfBytes);
      }
      __syncwarp();  // the stage is free for every lane, not only the one that waited
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      const size_t wt = weight_image(0, nt, kt, (p.NT + 1) / 2, p.KT);
      uint8_t* sb = smem + stage * C::kStageBytes;
      const bool sf = lane & 1;
      bulk_g2s_if(lane < 2, sf ? sb + C::kOffSfa : sb, sf ? p.Ws + wt * kTileSfBytes : p.Wq + wt * kTileCodeBytes,
                  sf ? kTileSfBytes : kTileCodeBytes, &full[stage]);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer ----
      // The scale copies come from warp 2: measured on this kernel, the hand-off costs
      // less than the slower MMA issue of a thread that mixes tcgen05.cp and waits.
      const uint32_t idesc_lo = idesc_mxf4(128, BT, 0, 0), idesc_hi = idesc_mxf4(128, BT, 2, 2);
      const uint64_t code0 = sdesc_kmajor_sw128(smem_u32(smem));
      bool ok = true;
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = kt0; kt < kt1; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag, kWaitTimeoutNs) ||
            !mbar_wait(&sfull[stage], phase, abort_flag, kWaitTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if constexpr (kDump) {
          if (nt == 0 && p.dump_codes != nullptr)
            dump_act_tile<BT>(smem + stage * C::kStageBytes + C::kOffB, smem + stage * C::kStageBytes + C::kOffSfb,
                              p, m0, rows, kt);
        }
        const uint32_t so = static_cast<uint32_t>(stage * C::kStageBytes) >> 4;
        const uint32_t sfa_col = tmem + C::kSfCol + 16 * stage;
        mma_stage(code0 + so, code0 + so + (C::kOffB >> 4), sfa_col, sfa_col + 8, tmem, idesc_lo, idesc_hi,
                  kt == kt0);
        tc_commit(&empty[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok) tc_commit(&accf[0]);
    }
  } else if (warp < 6) {
    // ---- during the mainloop, warp 2 copies each stage's scales into its TMEM slot (a
    // slot is rewritten only after its stage was refilled, which happens only after
    // the MMAs that read the slot completed); then the epilogue: FP32 partial tile to
    // local shared memory, then one bulk copy per owner ----
    const int q = warp & 3;
    const int et = threadIdx.x - 64;
    if (et == 0) {
      const uint64_t sf0 = sdesc_sf_block(smem_u32(smem));
      int stage = 0;
      uint32_t phase = 0;
      for (int kt = kt0; kt < kt1; ++kt) {
        if (!mbar_wait(&full[stage], phase, abort_flag, kWaitTimeoutNs)) break;
        const uint32_t so = static_cast<uint32_t>(stage * C::kStageBytes) >> 4;
        const uint32_t sfa_col = tmem + C::kSfCol + 16 * stage;
        scale_copies(sf0 + so + (C::kOffSfa >> 4), sf0 + so + (C::kOffSfb >> 4), sfa_col, sfa_col + 8);
        tc_commit(&sfull[stage]);
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
    __syncwarp();
    if (et == 0) *epi_flag = mbar_wait(&accf[0], 0, abort_flag, kWaitTimeoutNs) ? 1 : 0;
    named_bar_sync(1, 128);
    if (*epi_flag && !split) {
      // Without a K split the accumulator is the whole sum: each thread holds output
      // channel n0 + 32 q + lane for every token of the tile and stores it directly
      // (a warp writes 64 contiguous bytes of a y row per token).
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      const int n = nt * kRowsTile + q * 32 + lane;
      const float os = p.out_scale;
      float b = 0.f;
      if constexpr (kEpilogue) {
        if (p.bias != nullptr && n < p.N) b = __ldg(p.bias + n);
      }
      pdl_wait();  // y may still be read by the previous kernel on the stream
#pragma unroll 1
      for (int c0 = 0; c0 < BT; c0 += 16) {
        uint32_t r0[16];
        tmem_ld_32x32b_x16(taddr + c0, r0);
        tmem_wait_ld();
        if (n < p.N) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            if (c0 + jj >= rows) break;
            float v = __uint_as_float(r0[jj]) * os;
            if constexpr (kEpilogue) v = act_value_rt(v + b, p.act);
            const int64_t o = static_cast<int64_t>(m0 + c0 + jj) * p.N + n;
            if (p.y8 != nullptr) p.y8[o] = e4m3_1(v * p.y8_scale);
            else p.y[o] = bf16_bits(v);
          }
        }
      }
    } else if (*epi_flag) {
      tc_fence_after();
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16);
      float* col = part + q * 32 + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < BT; c0 += 32) {
        uint32_t r0[16], r1[16];
        tmem_ld_32x32b_x16(taddr + c0, r0);
        if (c0 + 16 < BT) tmem_ld_32x32b_x16(taddr + c0 + 16, r1);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) col[(c0 + jj) * kRowsTile] = __uint_as_float(r0[jj]);
        if (c0 + 16 < BT) {
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) col[(c0 + 16 + jj) * kRowsTile] = __uint_as_float(r1[jj]);
        }
      }
      fence_proxy_async_smem();
    }
    if (split) cluster_wait_acquire();  // every CTA runs and has its receive barrier armed
    cluster_waited = true;
    named_bar_sync(1, 128);
    if (split && *epi_flag && et == 0) {
      const uint32_t recv = smem_u32(smem + C::kRecvOff);
      const uint32_t slot = static_cast<uint32_t>(static_cast<int>(rank) * rpr * kRowsTile * 4);
      for (int o = 0; o < p.S; ++o) {
        const int n_rows = rows_of(o);
        if (n_rows == 0) continue;
        bulk_s2s_cluster(mapa_shared(recv + slot, static_cast<uint32_t>(o)), part + o * rpr * kRowsTile,
                         static_cast<uint32_t>(n_rows * kRowsTile * 4),
                         mapa_shared(smem_u32(recv_bar), static_cast<uint32_t>(o)));
      }
    }
  } else {
    // ---- activation prologue: x/D, FWHT32, BF16, E8M0, E2M1 -> swizzled B tile ----
    // the group's jj-th K tile: CTA-local index j = grp + kG * jj
    auto stage_body = [&](int jj, uint4 (&xv)[C::kTasks][4], const float (&d)[C::kRcp]) -> bool {
      const int j = grp + kG * jj, stage = j % kStages;
      const int slot = grp * 2 + (jj & 1);
      float* r = rbuf + slot * kQRcpTile;
#pragma unroll
      for (int e = 0; e < C::kRcp; ++e) r[qrcp_index(gt + e * kGT)] = __frcp_rn(d[e]);
      if (gt == 0) pro_flag[slot] = mbar_wait(&empty[stage], ((j / kStages) & 1) ^ 1, abort_flag, kWaitTimeoutNs) ? 1 : 0;
      named_bar_sync(2 + grp, kGT);
      if (!pro_flag[slot]) return false;
      uint8_t* bcode = smem + stage * C::kStageBytes + C::kOffB;
      uint8_t* bsf = smem + stage * C::kStageBytes + C::kOffSfb;
#pragma unroll
      for (int u = 0; u < C::kTasks; ++u) {
        const int task = gt + u * kGT, t = task >> 3, c = task & 7;
        uint4 cv;
        uint32_t sc;
        if (p.plain) {
          act_block_plain(xv[u], cv, sc);
        } else {
          float2 r2[16];
          load_rcp_block(r + c * kQRcpStride, r2);
          act_block(xv[u], r2, cv, sc);
        }
        *reinterpret_cast<uint4*>(bcode + code_chunk_offset(t, c)) = cv;
        bsf[sf_offset(t, c)] = static_cast<uint8_t>(sc);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&full[stage]);
      return true;
    };
    if (gst <= kAhead) {
#pragma unroll
      for (int jj = 0; jj < kAhead; ++jj) {
        if (jj >= gst) break;
        if (!stage_body(jj, xpre[jj], dpre[jj])) break;
      }
    } else if constexpr (C::kTasks >= 4) {
      // the largest token tile: registers hold one K tile of loads
      if (stage_body(0, xpre[0], dpre[0])) {
        uint4 xa[C::kTasks][4];
        float da[C::kRcp];
        for (int jj = 1; jj < gst; ++jj) {
          load(kt_of(jj), xa, da);
          if (!stage_body(jj, xa, da)) break;
        }
      }
    } else {
      // deeper K ranges: one K tile of loads ahead
      uint4 xa[C::kTasks][4], xb[C::kTasks][4];
      float da[C::kRcp], db[C::kRcp];
#pragma unroll
      for (int u = 0; u < C::kTasks; ++u)
#pragma unroll
        for (int i = 0; i < 4; ++i) xa[u][i] = xpre[0][u][i];
#pragma unroll
      for (int e = 0; e < C::kRcp; ++e) da[e] = dpre[0][e];
      if constexpr (kAhead >= 2) {
#pragma unroll
        for (int u = 0; u < C::kTasks; ++u)
#pragma unroll
          for (int i = 0; i < 4; ++i) xb[u][i] = xpre[1][u][i];
#pragma unroll
        for (int e = 0; e < C::kRcp; ++e) db[e] = dpre[1][e];
      }
      for (int jj = 0; jj < gst; jj += 2) {
        if (jj + 1 < gst && !(kAhead >= 2 && jj == 0)) load(kt_of(jj + 1), xb, db);
        if (!stage_body(jj, xa, da)) break;
        if (jj + 1 >= gst) break;
        if (jj + 2 < gst) load(kt_of(jj + 2), xa, da);
        if (!stage_body(jj + 1, xb, db)) break;
      }
    }
  }

  // ---- split-K reduction: wait for every rank's rows of this CTA, sum in rank order ----
  pdl_wait();  // y may still be read by the previous kernel on the stream
  __syncwarp();                                          // reconverge (warps 0 and 1 ran single-lane roles)
  if (split && !cluster_waited) cluster_wait_acquire();  // warp-uniform: the epilogue warps waited above
  if (split && threadIdx.x == 0) *epi_flag = mbar_wait(recv_bar, 0, abort_flag, kWaitTimeoutNs) ? 1 : 0;
  __syncthreads();
  if (*epi_flag && split) {  // (without a split the epilogue warps stored y already)
    const int t_lo = static_cast<int>(rank) * rpr, n_rows = rows_of(static_cast<int>(rank));
    const int n0 = nt * kRowsTile;
    // without a split the local partial tile is the whole sum
    const float* recv = split ? reinterpret_cast<const float*>(smem + C::kRecvOff) : part;
    for (int it = threadIdx.x; it < n_rows * 16; it += blockDim.x) {
      const int lr = it / 16, t = t_lo + lr, n = (it % 16) * 8;
      if (t >= rows || n0 + n >= p.N) continue;
      float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int src = 0; src < p.S; ++src) {  // fixed order: deterministic sums
        const float4* v = reinterpret_cast<const float4*>(recv + ((src * rpr + lr) * kRowsTile + n));
        const float4 a = v[0], b = v[1];
        s[0] += a.x; s[1] += a.y; s[2] += a.z; s[3] += a.w;
        s[4] += b.x; s[5] += b.y; s[6] += b.z; s[7] += b.w;
      }
      const float os = p.out_scale;
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] *= os;
      if constexpr (kEpilogue) {
        if (p.bias != nullptr) {
          const float4* b = reinterpret_cast<const float4*>(p.bias + n0 + n);
          const float4 b0 = __ldg(b), b1 = __ldg(b + 1);
          s[0] += b0.x; s[1] += b0.y; s[2] += b0.z; s[3] += b0.w;
          s[4] += b1.x; s[5] += b1.y; s[6] += b1.z; s[7] += b1.w;
        }
        if (p.act != 0) {
#pragma unroll
          for (int i = 0; i < 8; ++i) s[i] = act_value_rt(s[i], p.act);
        }
      }
      const int64_t off = static_cast<int64_t>(m0 + t) * p.N + n0 + n;
      if (p.y8 != nullptr) {
        const float2 sc = make_float2(p.y8_scale, p.y8_scale);
        uint2 o8;
        o8.x = e4m3x4(fmul2(make_float2(s[0], s[1]), sc), fmul2(make_float2(s[2], s[3]), sc));
        o8.y = e4m3x4(fmul2(make_float2(s[4], s[5]), sc), fmul2(make_float2(s[6], s[7]), sc));
        *reinterpret_cast<uint2*>(p.y8 + off) = o8;
      } else {
        uint4 o;
        o.x = pack_bf16x2(s[0], s[1]);
        o.y = pack_bf16x2(s[2], s[3]);
        o.z = pack_bf16x2(s[4], s[5]);
        o.w = pack_bf16x2(s[6], s[7]);
        *reinterpret_cast<uint4*>(p.y + off) = o;
      }
    }
  }
  // no CTA may leave while a copy it sent can still be reading its shared memory:
  // every rank arrives only after its own receive barrier completed
  if (split) {
    __syncwarp();
    cluster_arrive_release();
    cluster_wait_acquire();
  }

  if (*abort_flag && threadIdx.x == 0 && p.status) *p.status = MACAQ_ERR_DEVICE_TIMEOUT;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
}

}  // namespace macaq

// ============================================================================
// Host side: argument checks, variant choice, launches
// ============================================================================
using namespace macaq;

namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool probed = false;
  bool is_sm100 = false;
  int sms = 0;
  bool attrs_set = false;
};
DeviceState g_dev[kMaxDevices];

// Shared-memory opt-in of the fused kernel's instantiations for one token tile.
template <int BT>
bool fused_attrs() {
  const int bytes = fused::Cfg<BT>::kSmemBytes;
  const auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
  return cudaFuncSetAttribute(fused_small_kernel<BT, false, false>, a, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(fused_small_kernel<BT, true, false>, a, bytes) == cudaSuccess &&
         cudaFuncSetAttribute(fused_small_kernel<BT, false, true>, a, bytes) == cudaSuccess;
}

int current_device(int& dev, int& sms) {
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MACAQ_ERR_CUDA;
  DeviceState& s = g_dev[dev];
  if (!s.probed) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MACAQ_ERR_CUDA;
    s.is_sm100 = (major == 10 && minor == 0);
    s.sms = count;
    s.probed = true;
  }
  sms = s.sms;
  if (!s.is_sm100) return MACAQ_ERR_ARCH;
  if (!s.attrs_set) {  // once per device: opt in to the shared memory the kernels use
    const size_t gemm_smem = gemm::kSmemLimit;  // smem_bytes(E) stays within it for every E
    const auto a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    const int gs = static_cast<int>(gemm_smem);
    bool ok = cudaFuncSetAttribute(gemm_kernel<-1>, a, gs) == cudaSuccess &&
              cudaFuncSetAttribute(gemm_kernel<0>, a, gs) == cudaSuccess &&
              cudaFuncSetAttribute(gemm_kernel<1>, a, gs) == cudaSuccess &&
              cudaFuncSetAttribute(gemm_kernel<2>, a, gs) == cudaSuccess &&
              cudaFuncSetAttribute(gemm_kernel<4>, a, gs) == cudaSuccess &&
              cudaFuncSetAttribute(gemm_kernel<5>, a, gs) == cudaSuccess;
    ok = ok && fused_attrs<16>() && fused_attrs<32>() && fused_attrs<64>() && fused_attrs<128>();
    ok = ok && cudaFuncSetAttribute(quant_tiles_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kQuantSmem) ==
                   cudaSuccess;
    if (!ok) return MACAQ_ERR_CUDA;
    s.attrs_set = true;
  }
  return MACAQ_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na && nb && x < y + nb && y < x + na;
}

bool valid_nk(int64_t N, int64_t K) {
  return K >= 256 && K <= 65536 && K % 256 == 0 && N >= 16 && N <= 65536 && N % 16 == 0;
}

int64_t pad128(int64_t n) { return (n + 127) / 128 * 128; }
int64_t pad256(int64_t n) { return (n + 255) / 256 * 256; }
size_t align256(size_t n) { return (n + 255) / 256 * 256; }

template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, bool pdl,
                      int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attrs[2];
  int n = 0;
  if (pdl) {
    attrs[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  if (cluster_x > 1) {
    attrs[n].id = cudaLaunchAttributeClusterDimension;
    attrs[n].val.clusterDim.x = cluster_x;
    attrs[n].val.clusterDim.y = 1;
    attrs[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// ---- small-M fused plan: token tile BT and cluster size S ----
struct FusedPlan {
  int bt, S, ctas;
};

template <int BT>
int max_active_clusters(int S) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(S);
  cfg.blockDim = dim3(fused::kThreads);
  cfg.dynamicSmemBytes = fused::Cfg<BT>::kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = S;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, fused_small_kernel<BT>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int max_active_clusters_any(int bt_index, int S) {
  switch (bt_index) {
    case 0: return max_active_clusters<16>(S);
    case 1: return max_active_clusters<32>(S);
    case 2: return max_active_clusters<64>(S);
    default: return max_active_clusters<128>(S);
  }
}

// Co-resident clusters per (BT, S), measured once per device.
int active_clusters(int dev, int bt_index, int S) {
  static int cache[kMaxDevices][4][9] = {};
  int& v = cache[dev][bt_index][S];
  if (v == 0) {
    switch (bt_index) {
      case 0: v = max_active_clusters<16>(S); break;
      case 1: v = max_active_clusters<32>(S); break;
      case 2: v = max_active_clusters<64>(S); break;
      default: v = max_active_clusters<128>(S);
    }
    if (v <= 0) v = -1;  // query failed: treat as one cluster per wave
  }
  return v > 0 ? v : 1;
}

// Choose the token tile BT and the K split S (a divisor of K/256, at most 8
// CTAs per cluster) that minimise the time of a call, modelled per wave of
// clusters (µs, fitted to measured B200 timings of every feasible plan of the
// M = 16 and M = 128 workloads):
//   fixed 4.5 (launch, set-up, first loads, epilogue)
//   + max(prologue 0.55 per 16 rows per K tile, MMA issue 0.65 per K tile)
//     (the two overlap stage by stage; the slower sets the pace)
//   + split-K reduction 1.1 + 0.2 S when S > 1.
FusedPlan plan_fused(int dev, int64_t M, int64_t N, int64_t K) {
  const int NT = static_cast<int>(pad128(N) / 128), KT = static_cast<int>(K / 256);
  const int bts[4] = {16, 32, 64, 128};
  FusedPlan best{128, 1, 0};
  double best_cost = 1e30;
  for (int bi = 0; bi < 4; ++bi) {
    const int bt = bts[bi];
    if (bi > 0 && bts[bi - 1] >= M) break;  // a larger tile than M only adds empty rows
    const int clusters = NT * ceil_div(M, bt);
    for (int S = 1; S <= 8 && S <= KT; ++S) {
      if (KT % S) continue;
      const int waves = ceil_div(clusters, active_clusters(dev, bi, S));
      const double stages = static_cast<double>(KT / S), rows16 = static_cast<double>(M < bt ? M : bt) / 16.0;
      const double per_wave = 4.5 + std::max(0.55 * rows16 * stages, 0.65 * stages) + (S > 1 ? 1.1 + 0.2 * S : 0.0);
      const double cost = static_cast<double>(waves) * per_wave;
      if (cost <= best_cost + 1e-9) {  // on a tie the larger tile / split (measured faster)
        best_cost = cost;
        best = {bt, S, clusters * S};
      }
    }
  }
  return best;
}

template <bool kEpilogue, bool kDump = false>
cudaError_t launch_fused_kind(const FusedParams& p, const FusedPlan& plan, cudaStream_t st) {
  const dim3 grid(plan.ctas), block(fused::kThreads);
  switch (plan.bt) {
    case 16:
      return launch_ex(fused_small_kernel<16, kEpilogue, kDump>, grid, block, fused::Cfg<16>::kSmemBytes, st, true,
                       plan.S, p);
    case 32:
      return launch_ex(fused_small_kernel<32, kEpilogue, kDump>, grid, block, fused::Cfg<32>::kSmemBytes, st, true,
                       plan.S, p);
    case 64:
      return launch_ex(fused_small_kernel<64, kEpilogue, kDump>, grid, block, fused::Cfg<64>::kSmemBytes, st, true,
                       plan.S, p);
    default:
      return launch_ex(fused_small_kernel<128, kEpilogue, kDump>, grid, block, fused::Cfg<128>::kSmemBytes, st, true,
                       plan.S, p);
  }
}

int launch_fused(const FusedParams& p, const FusedPlan& plan, cudaStream_t st) {
  const cudaError_t e = (p.bias != nullptr || p.act != 0) ? launch_fused_kind<true>(p, plan, st)
                                                          : launch_fused_kind<false>(p, plan, st);
  return e == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

// ---- quantise-once workspace layouts ----
struct DenseWs {
  size_t act, total;
};
DenseWs dense_ws(int64_t M, int64_t K) {
  const size_t tiles = static_cast<size_t>(pad128(M) / 128) * (K / 256);
  DenseWs w;
  w.act = kWsReserved;
  w.total = w.act + tiles * kActImageBytes;
  return w;
}
struct GroupedWs {
  size_t goff, gtp, gexp, valid, slabs, act, total;
  int tiles_upper;
};
GroupedWs grouped_ws(int64_t M, int64_t K, int64_t E) {
  GroupedWs w;
  w.tiles_upper = static_cast<int>(pad128(M) / 128 + E);
  const size_t KT = K / 256;
  w.goff = kWsReserved;
  w.gtp = align256(w.goff + (E + 1) * 8);
  w.gexp = align256(w.gtp + (E + 1) * 4);
  w.valid = align256(w.gexp + E * 4);
  w.slabs = align256(w.valid + 16);  // valid flag, then the slab count
  w.act = align256(w.slabs + static_cast<size_t>((M + 31) / 32 + E) * 16);
  w.total = w.act + static_cast<size_t>(w.tiles_upper) * KT * kActImageBytes;
  return w;
}

// plain: plain MXFP4 call, D is not used (and may be null).
// weight_bytes: bytes of each of Wq and Ws when they are not prepared weights
// (the weight-list form passes tables of addresses); 0: prepared images of E experts.
// ybytes: bytes of the output (0: BF16 [M, N]).
int check_mm_args(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, void* y, int64_t M,
                  int64_t N, int64_t K, int64_t E, bool plain = false, size_t weight_bytes = 0, size_t ybytes = 0) {
  if (M < 0 || M > INT32_MAX || !valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (M == 0) return MACAQ_OK;
  if (!x || (!D && !plain) || !Wq || !Ws || !y) return MACAQ_ERR_NULL;
  if (!aligned16(x) || (!plain && !aligned16(D)) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y))
    return MACAQ_ERR_ALIGN;
  if (ybytes == 0) ybytes = static_cast<size_t>(M) * N * 2;
  if (overlaps(y, ybytes, x, static_cast<size_t>(M) * K * 2) ||
      (!plain && overlaps(y, ybytes, D, static_cast<size_t>(E) * K * 4)) ||
      overlaps(y, ybytes, Wq, weight_bytes ? weight_bytes : macaq_weight_code_bytes(E, N, K)) ||
      overlaps(y, ybytes, Ws, weight_bytes ? weight_bytes : macaq_weight_scale_bytes(E, N, K)))
    return MACAQ_ERR_ALIAS;
  return MACAQ_OK;
}

int check_ws(void* ws, size_t ws_bytes, size_t need, const void* y, size_t ybytes, const void* x, size_t xbytes) {
  if (!ws || ws_bytes < need || !aligned16(ws)) return MACAQ_ERR_WORKSPACE;
  if (overlaps(ws, need, y, ybytes) || overlaps(ws, need, x, xbytes)) return MACAQ_ERR_ALIAS;
  return MACAQ_OK;
}

// Quantiser grid: KT x per_kt CTAs, about kQuantCtasPerSm per SM, per_kt no
// more than the slabs (for grouped calls an upper bound of them).
int quant_grid(int64_t slabs, int KT, int sms) {
  int64_t per_kt = std::max<int64_t>(1, static_cast<int64_t>(sms) * kQuantCtasPerSm / KT);
  per_kt = std::min<int64_t>(per_kt, std::max<int64_t>(1, slabs));
  return static_cast<int>(per_kt * KT);
}

// Dense quantise-once: the quantiser over all rows, then the GEMM (launched as
// a programmatic dependent of the quantiser when `pdl`).
// Output epilogue of the _ex calls: fp32 bias (nullptr: none) and act_type.
struct Epilogue {
  const float* bias = nullptr;
  int act = 0;
  uint8_t* y8 = nullptr;  // FP8 (E4M3) output instead of BF16
  float y8_scale = 1.0f;
};
bool act_supported(int act) { return act == 0 || act == 1 || act == 2 || act == 4 || act == 5; }
// bias: 16-byte aligned, rows * N floats, not overlapping y.
int check_epilogue(const Epilogue& ep, int64_t rows, int64_t N, const void* y, size_t ybytes) {
  if (!act_supported(ep.act)) return MACAQ_ERR_ACT_TYPE;
  if (ep.bias == nullptr) return MACAQ_OK;
  if (!aligned16(ep.bias)) return MACAQ_ERR_ALIGN;
  if (overlaps(y, ybytes, ep.bias, static_cast<size_t>(rows) * N * 4)) return MACAQ_ERR_ALIAS;
  return MACAQ_OK;
}

// The GEMM instantiation for an epilogue: scaling only, or bias and act_type.
using GemmKernel = void (*)(GemmParams);
GemmKernel gemm_for(const float* bias, int act) {
  if (bias == nullptr && act == 0) return gemm_kernel<-1>;
  switch (act) {
    case 1: return gemm_kernel<1>;
    case 2: return gemm_kernel<2>;
    case 4: return gemm_kernel<4>;
    case 5: return gemm_kernel<5>;
    default: return gemm_kernel<0>;
  }
}

int run_dense_two_kernel(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y,
                         int64_t M, int64_t N, int64_t K, uint8_t* ws, int32_t* status, cudaStream_t st, int sms,
                         bool pdl, bool plain = false, Epilogue ep = Epilogue()) {
  const DenseWs w = dense_ws(M, K);
  const int MT = static_cast<int>(pad128(M) / 128), KT = static_cast<int>(K / 256);
  QuantParams qp{};
  qp.x = x; qp.D = D; qp.Aq = ws + w.act;
  qp.M = static_cast<int>(M); qp.K = static_cast<int>(K); qp.plain = plain ? 1 : 0;
  if (launch_ex(quant_tiles_kernel, dim3(quant_grid((M + 31) / 32, KT, sms)), dim3(256), kQuantSmem, st, pdl, 1,
                qp) !=
      cudaSuccess)
    return MACAQ_ERR_CUDA;
  GemmParams gp{};
  gp.Wq = Wq; gp.Ws = Ws; gp.Aq = qp.Aq; gp.y = y;
  gp.M = static_cast<int>(M); gp.N = static_cast<int>(N); gp.K = static_cast<int>(K);
  gp.NT = static_cast<int>(pad128(N) / 128); gp.KT = KT; gp.E = 1; gp.MT = MT;
  gp.NT2 = (gp.NT + 1) / 2; gp.stages = gemm::stages_for(0);
  gp.out_scale = plain ? 1.0f : 0.03125f;
  gp.bias = ep.bias;
  gp.act = ep.act;
  gp.y8 = ep.y8;
  gp.y8_scale = ep.y8_scale;
  gp.status = status;
  gp.wait_for_producer = pdl ? 1 : 0;
  const int tiles = MT * gp.NT2;
  const int grid = tiles < sms ? tiles : sms;
  const cudaError_t e =
      launch_ex(gemm_for(gp.bias, gp.act), dim3(grid),
                dim3(gemm::kThreads), gemm::smem_bytes(0), st, pdl, 1, gp);
  return e == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

// ---- scratch for callers that cannot allocate device memory ----
// One fixed buffer per device that loads this library, held until exit.  Host
// code must not hand the symbol itself to a kernel (in host code it names a
// host-side shadow); the device address is looked up once per device with
// that device current.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MACAQ_STATIC_SCRATCH_BYTES];

int noalloc_scratch(int dev, uint8_t** out) {
  static uint8_t* addr[kMaxDevices] = {};
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return MACAQ_ERR_CUDA;
    addr[dev] = static_cast<uint8_t*>(p);
  }
  *out = addr[dev];
  return MACAQ_OK;
}

}  // namespace

extern "C" {

const char* macaq_status_string(int s) {
  switch (s) {
    case MACAQ_OK: return "MACAQ_OK";
    case MACAQ_ERR_NULL: return "MACAQ_ERR_NULL";
    case MACAQ_ERR_ALIGN: return "MACAQ_ERR_ALIGN";
    case MACAQ_ERR_SHAPE: return "MACAQ_ERR_SHAPE";
    case MACAQ_ERR_ARCH: return "MACAQ_ERR_ARCH";
    case MACAQ_ERR_ALIAS: return "MACAQ_ERR_ALIAS";
    case MACAQ_ERR_TOO_MANY_GROUPS: return "MACAQ_ERR_TOO_MANY_GROUPS";
    case MACAQ_ERR_GROUP_LIST_TYPE: return "MACAQ_ERR_GROUP_LIST_TYPE";
    case MACAQ_ERR_CUDA: return "MACAQ_ERR_CUDA";
    case MACAQ_ERR_DEVICE_TIMEOUT: return "MACAQ_ERR_DEVICE_TIMEOUT";
    case MACAQ_ERR_GROUP_LIST_INVALID: return "MACAQ_ERR_GROUP_LIST_INVALID";
    case MACAQ_ERR_WORKSPACE: return "MACAQ_ERR_WORKSPACE";
    case MACAQ_ERR_BAD_D: return "MACAQ_ERR_BAD_D";
    case MACAQ_ERR_ACT_TYPE: return "MACAQ_ERR_ACT_TYPE";
    default: return "MACAQ_ERR_UNKNOWN";
  }
}

int macaq_abi_version(void) { return MACAQ_ABI_VERSION; }

size_t macaq_weight_code_bytes(int64_t E, int64_t N, int64_t K) {
  if (E < 1 || E > kMaxGroups || !valid_nk(N, K)) return 0;
  return static_cast<size_t>(E) * pad256(N) * (K / 2);
}

size_t macaq_weight_scale_bytes(int64_t E, int64_t N, int64_t K) {
  if (E < 1 || E > kMaxGroups || !valid_nk(N, K)) return 0;
  return static_cast<size_t>(E) * pad256(N) * (K / 32);
}

static int prepare_impl(const float* W, const float* D, int64_t E, int64_t N, int64_t K, uint8_t* Wq, uint8_t* Ws,
                        void* stream, bool trans);

int macaq_prepare_weights(const float* W, const float* D, int64_t E, int64_t N, int64_t K, uint8_t* Wq, uint8_t* Ws,
                          void* stream) {
  return prepare_impl(W, D, E, N, K, Wq, Ws, stream, false);
}

int macaq_prepare_weights_transposed(const float* W_kn, const float* D, int64_t E, int64_t N, int64_t K, uint8_t* Wq,
                                     uint8_t* Ws, void* stream) {
  return prepare_impl(W_kn, D, E, N, K, Wq, Ws, stream, true);
}

static int prepare_impl(const float* W, const float* D, int64_t E, int64_t N, int64_t K, uint8_t* Wq, uint8_t* Ws,
                        void* stream, bool trans) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (!valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (!W || !D || !Wq || !Ws) return MACAQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(D) || !aligned16(Wq) || !aligned16(Ws)) return MACAQ_ERR_ALIGN;
  const size_t qb = macaq_weight_code_bytes(E, N, K), sb = macaq_weight_scale_bytes(E, N, K);
  const size_t wb = static_cast<size_t>(E * N * K * 4), db = static_cast<size_t>(E * K * 4);
  if (overlaps(Wq, qb, W, wb) || overlaps(Wq, qb, D, db) || overlaps(Ws, sb, W, wb) || overlaps(Ws, sb, D, db) ||
      overlaps(Wq, qb, Ws, sb))
    return MACAQ_ERR_ALIAS;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // D must be finite and nonzero: read it back once (this call is offline).
  std::vector<float> hD(static_cast<size_t>(E * K));
  if (cudaMemcpyAsync(hD.data(), D, hD.size() * sizeof(float), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MACAQ_ERR_CUDA;
  for (float d : hD)
    if (!(d != 0.0f) || !std::isfinite(d)) return MACAQ_ERR_BAD_D;
  const int NTP = static_cast<int>(pad256(N) / 128);  // images per expert, pairs complete
  dim3 grid(static_cast<unsigned>(E * NTP * 4), static_cast<unsigned>(K / 256));
  if (trans)
    prep_weights_kernel<false, true><<<grid, 256, 0, s>>>(W, D, Wq, Ws, static_cast<int>(N), static_cast<int>(K), NTP);
  else
    prep_weights_kernel<false, false><<<grid, 256, 0, s>>>(W, D, Wq, Ws, static_cast<int>(N), static_cast<int>(K), NTP);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_prepare_weights_plain(const float* W, int64_t E, int64_t N, int64_t K, uint8_t* Wq, uint8_t* Ws,
                                void* stream) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (!valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (!W || !Wq || !Ws) return MACAQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(Ws)) return MACAQ_ERR_ALIGN;
  const size_t qb = macaq_weight_code_bytes(E, N, K), sb = macaq_weight_scale_bytes(E, N, K);
  const size_t wb = static_cast<size_t>(E * N * K * 4);
  if (overlaps(Wq, qb, W, wb) || overlaps(Ws, sb, W, wb) || overlaps(Wq, qb, Ws, sb)) return MACAQ_ERR_ALIAS;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const int NTP = static_cast<int>(pad256(N) / 128);
  dim3 grid(static_cast<unsigned>(E * NTP * 4), static_cast<unsigned>(K / 256));
  prep_weights_kernel<true><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      W, nullptr, Wq, Ws, static_cast<int>(N), static_cast<int>(K), NTP);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

size_t macaq_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E) {
  if (M <= 0 || !valid_nk(N, K) || E < 1 || E > kMaxGroups) return 0;
  if (E > 1) return grouped_ws(M, K, E).total;
  if (M <= kSmallM) return 0;
  return dense_ws(M, K).total;
}

static int dense_impl(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y, int64_t M,
               int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream, bool plain,
               Epilogue ep = Epilogue()) {
  int st = check_mm_args(x, D, Wq, Ws, y, M, N, K, 1, plain);
  if (st == MACAQ_OK) st = check_epilogue(ep, 1, N, y, static_cast<size_t>(M) * N * 2);
  if (st != MACAQ_OK || M == 0) return st;
  if (M > kSmallM) {
    st = check_ws(workspace, workspace_bytes, dense_ws(M, K).total, y, static_cast<size_t>(M) * N * 2, x,
                  static_cast<size_t>(M) * K * 2);
    if (st != MACAQ_OK) return st;
  }
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M <= kSmallM) {
    FusedParams p{};
    p.Wq = Wq; p.Ws = Ws; p.x = x; p.D = D; p.y = y;
    p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
    p.NT = static_cast<int>(pad128(N) / 128); p.KT = static_cast<int>(K / 256);
    const FusedPlan plan = plan_fused(dev, M, N, K);
    p.S = plan.S;
    p.status = status;
    p.plain = plain ? 1 : 0;
    p.out_scale = plain ? 1.0f : 0.03125f;
    p.bias = ep.bias;
    p.act = ep.act;
    return launch_fused(p, plan, s);
  }
  return run_dense_two_kernel(x, D, Wq, Ws, y, M, N, K, static_cast<uint8_t*>(workspace), status, s, sms, true,
                              plain, ep);
}

// Weight-list form: device tables of E image addresses (see WeightList).
struct ListArg {
  const uint64_t* wq = nullptr;
  const uint64_t* ws = nullptr;
};

static int grouped_impl(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, const int64_t* group_list,
                 int group_list_type, int64_t E, uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                 size_t workspace_bytes, int32_t* status, void* stream, bool plain, Epilogue ep = Epilogue(),
                 ListArg list = ListArg()) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (group_list_type < 0 || group_list_type > 2) return MACAQ_ERR_GROUP_LIST_TYPE;
  const bool listed = list.wq != nullptr || list.ws != nullptr;
  void* yout = ep.y8 != nullptr ? static_cast<void*>(ep.y8) : static_cast<void*>(y);
  const size_t ybytes = static_cast<size_t>(M) * N * (ep.y8 != nullptr ? 1 : 2);
  int st;
  if (!listed) {
    st = check_mm_args(x, D, Wq, Ws, yout, M, N, K, E, plain, 0, ybytes);
  } else {  // the tables are checked here, the addresses in them on the device (group_tables_kernel)
    st = check_mm_args(x, D, reinterpret_cast<const uint8_t*>(list.wq), reinterpret_cast<const uint8_t*>(list.ws),
                       yout, M, N, K, E, plain, /*weight_bytes=*/static_cast<size_t>(E) * 8, ybytes);
  }
  if (st == MACAQ_OK) st = check_epilogue(ep, E, N, yout, ybytes);
  if (st != MACAQ_OK) return st;
  if (M == 0) return MACAQ_OK;
  if (!group_list) return MACAQ_ERR_NULL;
  if (!aligned16(group_list)) return MACAQ_ERR_ALIGN;
  const size_t gl_bytes = static_cast<size_t>(E) * (group_list_type == 2 ? 16 : 8);
  if (overlaps(yout, ybytes, group_list, gl_bytes)) return MACAQ_ERR_ALIAS;
  const GroupedWs w = grouped_ws(M, K, E);
  st = check_ws(workspace, workspace_bytes, w.total, yout, ybytes, x, static_cast<size_t>(M) * K * 2);
  if (st != MACAQ_OK) return st;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int64_t* goff = reinterpret_cast<int64_t*>(ws + w.goff);
  int* gtp = reinterpret_cast<int*>(ws + w.gtp);
  int* valid = reinterpret_cast<int*>(ws + w.valid);
  int4* slabs = reinterpret_cast<int4*>(ws + w.slabs);
  int* gexp = reinterpret_cast<int*>(ws + w.gexp);
  WeightList wl{};
  if (listed) {
    wl.wq = list.wq;
    wl.ws = list.ws;
    wl.wq_bytes = macaq_weight_code_bytes(1, N, K);
    wl.ws_bytes = macaq_weight_scale_bytes(1, N, K);
    wl.y_lo = reinterpret_cast<uint64_t>(yout);
    wl.y_hi = wl.y_lo + ybytes;
  }
  group_tables_kernel<<<1, static_cast<unsigned>((E + 31) / 32 * 32), 0, s>>>(
      group_list, group_list_type, static_cast<int>(E), static_cast<int>(M), goff, gtp, gexp, slabs, valid + 1, valid,
      status, wl);
  if (cudaPeekAtLastError() != cudaSuccess) return MACAQ_ERR_CUDA;
  const int KT = static_cast<int>(K / 256);
  QuantParams qp{};
  qp.x = x; qp.D = D; qp.Aq = ws + w.act;
  qp.M = static_cast<int>(M); qp.K = static_cast<int>(K);
  qp.slabs = slabs; qp.nslabs = valid + 1; qp.valid = valid; qp.plain = plain ? 1 : 0;
  if (launch_ex(quant_tiles_kernel, dim3(quant_grid((M + 31) / 32 + E, KT, sms)), dim3(256), kQuantSmem, s, true,
                1, qp) != cudaSuccess)
    return MACAQ_ERR_CUDA;
  GemmParams gp{};
  gp.Wq = Wq; gp.Ws = Ws; gp.Aq = qp.Aq; gp.y = y;
  gp.M = static_cast<int>(M); gp.N = static_cast<int>(N); gp.K = static_cast<int>(K);
  gp.NT = static_cast<int>(pad128(N) / 128); gp.KT = KT; gp.E = static_cast<int>(E);
  gp.NT2 = (gp.NT + 1) / 2; gp.stages = gemm::stages_for(static_cast<int>(E), listed);
  gp.goff = goff; gp.gtp = gtp; gp.gexp = gexp; gp.valid = valid;
  gp.out_scale = plain ? 1.0f : 0.03125f;
  gp.bias = ep.bias;
  gp.act = ep.act;
  gp.status = status;
  gp.wq_list = list.wq;
  gp.ws_list = list.ws;
  gp.y8 = ep.y8;
  gp.y8_scale = ep.y8_scale;
  const cudaError_t e = launch_ex(gemm_for(gp.bias, gp.act),
                                  dim3(sms), dim3(gemm::kThreads),
                                  gemm::smem_bytes(static_cast<int>(E), listed), s, true, 1, gp);
  return e == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_dense_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y, int64_t M,
                   int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return dense_impl(x, D, Wq, Ws, y, M, N, K, workspace, workspace_bytes, status, stream, false);
}

int macaq_dense_mm_ex(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, const float* bias,
                      int act_type, uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace,
                      size_t workspace_bytes, int32_t* status, void* stream) {
  Epilogue ep;
  ep.bias = bias;
  ep.act = act_type;
  return dense_impl(x, D, Wq, Ws, y, M, N, K, workspace, workspace_bytes, status, stream, false, ep);
}

int macaq_grouped_mm_ex(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws,
                        const int64_t* group_list, int group_list_type, int64_t E, const float* bias, int act_type,
                        uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                        int32_t* status, void* stream) {
  Epilogue ep;
  ep.bias = bias;
  ep.act = act_type;
  return grouped_impl(x, D, Wq, Ws, group_list, group_list_type, E, y, M, N, K, workspace, workspace_bytes, status,
                      stream, false, ep);
}

int macaq_dense_mm_fp8(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, const float* bias,
                       int act_type, float y_scale, uint8_t* y8, int64_t M, int64_t N, int64_t K, void* workspace,
                       size_t workspace_bytes, int32_t* status, void* stream) {
  Epilogue ep;
  ep.bias = bias;
  ep.act = act_type;
  ep.y8 = y8;
  ep.y8_scale = y_scale;
  const size_t ybytes = static_cast<size_t>(M) * N;
  int st = check_mm_args(x, D, Wq, Ws, y8, M, N, K, 1, false, 0, ybytes);
  if (st == MACAQ_OK) st = check_epilogue(ep, 1, N, y8, ybytes);
  if (st == MACAQ_OK && !(std::isfinite(y_scale) && y_scale > 0.0f)) st = MACAQ_ERR_SHAPE;
  if (st != MACAQ_OK || M == 0) return st;
  st = check_ws(workspace, workspace_bytes, dense_ws(M, K).total, y8, ybytes, x, static_cast<size_t>(M) * K * 2);
  if (st != MACAQ_OK) return st;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  if (M <= kSmallM) {  // the fused kernel, as macaq_dense_mm_ex, storing E4M3 codes
    FusedParams p{};
    p.Wq = Wq; p.Ws = Ws; p.x = x; p.D = D; p.y = nullptr;
    p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
    p.NT = static_cast<int>(pad128(N) / 128); p.KT = static_cast<int>(K / 256);
    const FusedPlan plan = plan_fused(dev, M, N, K);
    p.S = plan.S;
    p.status = status;
    p.out_scale = 0.03125f;
    p.bias = bias;
    p.act = act_type;
    p.y8 = y8;
    p.y8_scale = y_scale;
    return launch_fused(p, plan, static_cast<cudaStream_t>(stream));
  }
  return run_dense_two_kernel(x, D, Wq, Ws, nullptr, M, N, K, static_cast<uint8_t*>(workspace), status,
                              static_cast<cudaStream_t>(stream), sms, true, false, ep);
}

int macaq_grouped_mm_fp8(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws,
                         const int64_t* group_list, int group_list_type, int64_t E, const float* bias, int act_type,
                         float y_scale, uint8_t* y8, int64_t M, int64_t N, int64_t K, void* workspace,
                         size_t workspace_bytes, int32_t* status, void* stream) {
  if (!(std::isfinite(y_scale) && y_scale > 0.0f)) return MACAQ_ERR_SHAPE;
  Epilogue ep;
  ep.bias = bias;
  ep.act = act_type;
  ep.y8 = y8;
  ep.y8_scale = y_scale;
  return grouped_impl(x, D, Wq, Ws, group_list, group_list_type, E, nullptr, M, N, K, workspace, workspace_bytes,
                      status, stream, false, ep);
}

int macaq_grouped_mm_list(const uint16_t* x, const float* D, const uint64_t* Wq_list, const uint64_t* Ws_list,
                          const int64_t* group_list, int group_list_type, int64_t E, const float* bias, int act_type,
                          uint16_t* y, int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes,
                          int32_t* status, void* stream) {
  Epilogue ep;
  ep.bias = bias;
  ep.act = act_type;
  ListArg list;
  list.wq = Wq_list;
  list.ws = Ws_list;
  return grouped_impl(x, D, nullptr, nullptr, group_list, group_list_type, E, y, M, N, K, workspace, workspace_bytes,
                      status, stream, false, ep, list);
}

int macaq_calibrate_d(const uint16_t* x, int64_t T, const float* W, int64_t E, int64_t N, int64_t K,
                      const int64_t* group_list, int group_list_type, float* D, void* stream) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (T < 0 || T > INT32_MAX || N < 1 || N > 65536 || K < 256 || K > 65536 || K % 256) return MACAQ_ERR_SHAPE;
  if (!W || !D || (T > 0 && !x) || (!group_list && E != 1)) return MACAQ_ERR_NULL;
  if (group_list && (group_list_type < 0 || group_list_type > 2)) return MACAQ_ERR_GROUP_LIST_TYPE;
  if ((x && !aligned16(x)) || !aligned16(W) || !aligned16(D) || (group_list && !aligned16(group_list)))
    return MACAQ_ERR_ALIGN;
  const size_t dbytes = static_cast<size_t>(E) * K * 4;
  const size_t gl_len = group_list ? static_cast<size_t>(E) * (group_list_type == 2 ? 2 : 1) : 0;
  if (overlaps(D, dbytes, x, static_cast<size_t>(T) * K * 2) || overlaps(D, dbytes, W, static_cast<size_t>(E) * N * K * 4) ||
      overlaps(D, dbytes, group_list, gl_len * 8))
    return MACAQ_ERR_ALIAS;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (group_list) {  // offline: read the list back and check it (npu_grouped_matmul's group_list rules)
    std::vector<int64_t> h(gl_len);
    if (cudaMemcpyAsync(h.data(), group_list, gl_len * 8, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return MACAQ_ERR_CUDA;
    int64_t total = 0, prev = 0;
    for (int64_t j = 0; j < E; ++j) {
      int64_t cnt;
      if (group_list_type == 2) {
        if (h[2 * j] < 0 || h[2 * j] >= E) return MACAQ_ERR_GROUP_LIST_INVALID;
        cnt = h[2 * j + 1];
      } else if (group_list_type == 1) {
        cnt = h[j];
      } else {
        if (h[j] < prev) return MACAQ_ERR_GROUP_LIST_INVALID;
        cnt = h[j] - prev;
        prev = h[j];
      }
      if (cnt < 0 || cnt > T) return MACAQ_ERR_GROUP_LIST_INVALID;
      total += cnt;
      if (total > T) return MACAQ_ERR_GROUP_LIST_INVALID;
    }
    if (total != T) return MACAQ_ERR_GROUP_LIST_INVALID;
  }
  CalibParams p{};
  p.x = x; p.W = W; p.gl = group_list; p.type = group_list_type;
  p.E = static_cast<int>(E); p.N = static_cast<int>(N); p.K = static_cast<int>(K); p.T = T; p.D = D;
  const cudaError_t e = launch_ex(calibrate_kernel,
                                  dim3(static_cast<unsigned>(K / kCalibCols * kCalibCluster), static_cast<unsigned>(E)),
                                  dim3(1024), 0, s, false, kCalibCluster, p);
  return e == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_dense_mm_plain(const uint16_t* x, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y, int64_t M, int64_t N,
                         int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return dense_impl(x, nullptr, Wq, Ws, y, M, N, K, workspace, workspace_bytes, status, stream, true);
}

int macaq_grouped_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws,
                     const int64_t* group_list, int group_list_type, int64_t E, uint16_t* y, int64_t M, int64_t N,
                     int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return grouped_impl(x, D, Wq, Ws, group_list, group_list_type, E, y, M, N, K, workspace, workspace_bytes, status,
                      stream, false);
}

int macaq_grouped_mm_plain(const uint16_t* x, const uint8_t* Wq, const uint8_t* Ws, const int64_t* group_list,
                           int group_list_type, int64_t E, uint16_t* y, int64_t M, int64_t N, int64_t K,
                           void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  return grouped_impl(x, nullptr, Wq, Ws, group_list, group_list_type, E, y, M, N, K, workspace, workspace_bytes,
                      status, stream, true);
}

int macaq_quantize_activations(const uint16_t* x, const float* D, uint8_t* codes, uint8_t* scales, int64_t M,
                               int64_t K, void* stream) {
  if (M < 0 || M > INT32_MAX || K < 256 || K > 65536 || K % 256) return MACAQ_ERR_SHAPE;
  if (M == 0) return MACAQ_OK;
  if (!x || !D || !codes || !scales) return MACAQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(D) || !aligned16(codes) || !aligned16(scales)) return MACAQ_ERR_ALIGN;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  dim3 grid(static_cast<unsigned>((M + 31) / 32), static_cast<unsigned>(K / 256));
  quant_canonical_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, D, codes, scales, static_cast<int>(M), static_cast<int>(K));
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_export_weights(const uint8_t* Wq, const uint8_t* Ws, uint8_t* codes, uint8_t* scales, int64_t E, int64_t N,
                         int64_t K, void* stream) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (!valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (!Wq || !Ws || !codes || !scales) return MACAQ_ERR_NULL;
  if (!aligned16(Wq) || !aligned16(codes)) return MACAQ_ERR_ALIGN;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  dim3 grid(static_cast<unsigned>((E * N + 31) / 32), static_cast<unsigned>(K / 256));
  export_tiles_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      Wq, Ws, codes, scales, static_cast<int>(N), static_cast<int>(K), static_cast<int>(pad256(N) / 256),
      static_cast<int>(E * N));
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_mx_encode_blocks(const float* v, uint8_t* codes, uint8_t* scales, int64_t n, void* stream) {
  if (n < 0 || n % 32) return MACAQ_ERR_SHAPE;
  if (n == 0) return MACAQ_OK;
  if (!v || !codes || !scales) return MACAQ_ERR_NULL;
  if (!aligned16(v) || !aligned16(codes)) return MACAQ_ERR_ALIGN;
  int dev, sms;
  int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const int64_t nb = n / 32;
  mx_encode_kernel<<<static_cast<unsigned>((nb + 255) / 256), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      v, codes, scales, nb);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

size_t macaq_unfused_workspace_bytes(int64_t M, int64_t K) {
  if (M <= 0 || K < 256 || K > 65536 || K % 256) return 0;
  return dense_ws(M, K).total;
}

int macaq_dense_mm_noalloc(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y,
                           int64_t M, int64_t N, int64_t K, int32_t* status, void* stream) {
  int st = check_mm_args(x, D, Wq, Ws, y, M, N, K, 1);
  if (st != MACAQ_OK || M == 0) return st;
  if (dense_ws(M, K).total > MACAQ_STATIC_SCRATCH_BYTES) return MACAQ_ERR_WORKSPACE;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  uint8_t* scratch = nullptr;
  st = noalloc_scratch(dev, &scratch);
  if (st != MACAQ_OK) return st;
  return run_dense_two_kernel(x, D, Wq, Ws, y, M, N, K, scratch, status, static_cast<cudaStream_t>(stream), sms,
                              true);
}

int macaq_fused_plan(int64_t M, int64_t N, int64_t K, int* token_tile, int* k_split) {
  if (M < 1 || M > kSmallM || !valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (!token_tile || !k_split) return MACAQ_ERR_NULL;
  int dev, sms;
  const int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const FusedPlan plan = plan_fused(dev, M, N, K);
  *token_tile = plan.bt;
  *k_split = plan.S;
  return MACAQ_OK;
}

int macaq_fused_probe(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y, int64_t M,
                      int64_t N, int64_t K, int token_tile, int k_split, int plain, uint8_t* codes, uint8_t* scales,
                      int32_t* status, void* stream) {
  const bool pl = plain != 0;
  int st = check_mm_args(x, D, Wq, Ws, y, M, N, K, 1, pl);
  if (st != MACAQ_OK || M == 0) return st;
  const int KT = static_cast<int>(K / 256);
  if (M > kSmallM || (token_tile != 16 && token_tile != 32 && token_tile != 64 && token_tile != 128) ||
      k_split < 1 || k_split > 8 || KT % k_split != 0)
    return MACAQ_ERR_SHAPE;
  if ((codes == nullptr) != (scales == nullptr)) return MACAQ_ERR_NULL;
  if (codes != nullptr) {
    if (!aligned16(codes)) return MACAQ_ERR_ALIGN;
    const size_t cb = static_cast<size_t>(M) * K / 2, sb = static_cast<size_t>(M) * K / 32, yb = static_cast<size_t>(M) * N * 2;
    if (overlaps(codes, cb, y, yb) || overlaps(scales, sb, y, yb) || overlaps(codes, cb, scales, sb) ||
        overlaps(codes, cb, x, static_cast<size_t>(M) * K * 2) || overlaps(scales, sb, x, static_cast<size_t>(M) * K * 2))
      return MACAQ_ERR_ALIAS;
  }
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const int bi = token_tile == 16 ? 0 : token_tile == 32 ? 1 : token_tile == 64 ? 2 : 3;
  if (k_split > 1 && max_active_clusters_any(bi, k_split) < 1) return MACAQ_ERR_SHAPE;
  const FusedPlan plan{token_tile, k_split, static_cast<int>(pad128(N) / 128) * ceil_div(M, token_tile) * k_split};
  FusedParams p{};
  p.Wq = Wq; p.Ws = Ws; p.x = x; p.D = D; p.y = y;
  p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
  p.NT = static_cast<int>(pad128(N) / 128); p.KT = KT;
  p.S = k_split;
  p.status = status;
  p.plain = pl ? 1 : 0;
  p.out_scale = pl ? 1.0f : 0.03125f;
  p.dump_codes = codes;
  p.dump_scales = scales;
  // without a copy the product instantiation runs, exactly as macaq_dense_mm would run this plan
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = codes != nullptr ? launch_fused_kind<false, true>(p, plan, s) : launch_fused_kind<false, false>(p, plan, s);
  return e == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_test_wait_expiry(int64_t timeout_ns, int32_t* status, void* stream) {
  if (timeout_ns < 1000 || timeout_ns > 1000000000) return MACAQ_ERR_SHAPE;
  if (!status) return MACAQ_ERR_NULL;
  if (!aligned16(status)) return MACAQ_ERR_ALIGN;
  int dev, sms;
  const int st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  wait_expiry_kernel<<<1, 64, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint64_t>(timeout_ns), status);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int macaq_unfused_dense_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y,
                           int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int32_t* status,
                           void* stream) {
  int st = check_mm_args(x, D, Wq, Ws, y, M, N, K, 1);
  if (st != MACAQ_OK || M == 0) return st;
  st = check_ws(workspace, workspace_bytes, dense_ws(M, K).total, y, static_cast<size_t>(M) * N * 2, x,
                static_cast<size_t>(M) * K * 2);
  if (st != MACAQ_OK) return st;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  return run_dense_two_kernel(x, D, Wq, Ws, y, M, N, K, static_cast<uint8_t*>(workspace), status,
                              static_cast<cudaStream_t>(stream), sms, false);
}

}  // extern "C"
