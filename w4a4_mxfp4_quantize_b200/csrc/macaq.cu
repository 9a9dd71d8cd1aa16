// B200 (sm_100a) MACAQ W4A4 MXFP4 linear: kernels and the C ABI of macaq.h.
//
// Kernels
//   prep_weights_kernel   offline: W*D -> FWHT32 -> MX -> tensor-core tile images
//   quant_act_kernel      activation prologue alone (canonical or tiled output)
//   mma_kernel<BT,F>      the hot path: persistent, warp-specialised
//       warp 0      bulk-copy producer (TMA engine) of weight code/scale tiles
//                   (and of pre-quantised activation tiles when F = false)
//       warp 1      TMEM owner and single-thread tcgen05.mma kind::mxf4 issuer
//       warps 2-5   epilogue: tcgen05.ld -> x 2^-5 -> BF16 -> global
//                   (or FP32 split-K partials + in-kernel ordered reduction)
//       warps 6-13  (F = true) activation prologue: x/D, FWHT32, BF16, E8M0,
//                   E2M1 written straight into the swizzled shared-memory
//                   operand tile and its scale image
//   The MMA is swapped: the weight tile (128 output channels) is operand A,
//   the activation tile (BT tokens) is operand B, so small token counts map to
//   the narrow N side of the instruction (N = BT in {16, 32, 64, 128}).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "macaq.h"
#include "mx.cuh"
#include "ptx.cuh"

namespace macaq {

constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bounded waits give up after 2 s
constexpr int kStages = 4;
constexpr int kMaxGroups = 1024;

__host__ __device__ constexpr int ceil_div(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

// ============================================================================
// Offline weight preparation
// ============================================================================
// CTA = 32 rows x one 256-wide K tile (256 threads, one 32-block each).
__global__ void __launch_bounds__(256) prep_weights_kernel(const float* __restrict__ W, const float* __restrict__ D,
                                                           uint8_t* __restrict__ Wq, uint8_t* __restrict__ Ws,
                                                           int N, int K, int NT) {
  const int KT = K / kKTile;
  const int kt = blockIdx.y;
  const int t = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int row_global = blockIdx.x * 32 + t;  // over E * NT * 128 padded rows
  const int e = row_global / (NT * kRowsTile);
  const int rpad = row_global % (NT * kRowsTile);
  const int nt = rpad / kRowsTile, r = rpad % kRowsTile;
  const int n = rpad;
  const int64_t k0 = static_cast<int64_t>(kt) * kKTile + c * kBlk;
  uint4 codes = make_uint4(0, 0, 0, 0);
  uint32_t scale = 0;
  if (n < N) {
    float wv[32], dv[32];
    const float4* wp = reinterpret_cast<const float4*>(W + (static_cast<int64_t>(e) * N + n) * K + k0);
    const float4* dp = reinterpret_cast<const float4*>(D + static_cast<int64_t>(e) * K + k0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 a = __ldg(wp + i), b = __ldg(dp + i);
      wv[4 * i] = a.x; wv[4 * i + 1] = a.y; wv[4 * i + 2] = a.z; wv[4 * i + 3] = a.w;
      dv[4 * i] = b.x; dv[4 * i + 1] = b.y; dv[4 * i + 2] = b.z; dv[4 * i + 3] = b.w;
    }
    weight_block(wv, dv, codes, scale);
  }
  const size_t tile = (static_cast<size_t>(e) * NT + nt) * KT + kt;
  *reinterpret_cast<uint4*>(Wq + tile * kTileCodeBytes + code_chunk_offset(r, c)) = codes;
  Ws[tile * kTileSfBytes + sf_offset(r, c)] = static_cast<uint8_t>(scale);
}

// Tiled images -> canonical row-major codes/scales (tests only).
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
  const size_t tile = (static_cast<size_t>(e) * RT + nt) * KT + kt;
  const uint4 v = *reinterpret_cast<const uint4*>(Tq + tile * kTileCodeBytes + code_chunk_offset(r, c));
  const uint8_t s = Ts[tile * kTileSfBytes + sf_offset(r, c)];
  const int64_t row = static_cast<int64_t>(e) * R + n;
  *reinterpret_cast<uint4*>(codes + row * (K / 2) + (kt * kKTile + c * kBlk) / 2) = v;
  scales[row * (K / kBlk) + kt * (kKTile / kBlk) + c] = s;
}

// ============================================================================
// Standalone activation quantisation (test path and unfused ablation)
// ============================================================================
// CTA = 32 rows x one K tile, 256 threads.  kTiled: write 128-row tile images
// (rows >= M of the last tile get zero codes); else canonical [M, K/2].
template <bool kTiled>
__global__ void __launch_bounds__(256) quant_act_kernel(const uint16_t* __restrict__ x, const float* __restrict__ D,
                                                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                        int M, int K, int M_out) {
  __shared__ float r[kKTile];
  const int kt = blockIdx.y;
  const int64_t k0 = static_cast<int64_t>(kt) * kKTile;
  r[threadIdx.x] = __frcp_rn(__ldg(D + k0 + threadIdx.x));
  __syncthreads();
  const int t = threadIdx.x >> 3, c = threadIdx.x & 7;
  const int m = blockIdx.x * 32 + t;
  if (m >= M_out) return;
  uint4 cv = make_uint4(0, 0, 0, 0);
  uint32_t sc = 0;
  if (m < M) {
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(m) * K + k0 + c * kBlk);
    uint4 xv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = __ldg(src + i);
    act_block(xv, r + c * kBlk, cv, sc);
  }
  if constexpr (kTiled) {
    const int KT = K / kKTile;
    const size_t tile = static_cast<size_t>(m / kRowsTile) * KT + kt;
    const uint32_t rr = m % kRowsTile;
    *reinterpret_cast<uint4*>(codes + tile * kTileCodeBytes + code_chunk_offset(rr, c)) = cv;
    scales[tile * kTileSfBytes + sf_offset(rr, c)] = static_cast<uint8_t>(sc);
  } else {
    *reinterpret_cast<uint4*>(codes + static_cast<int64_t>(m) * (K / 2) + (k0 + c * kBlk) / 2) = cv;
    scales[static_cast<int64_t>(m) * (K / kBlk) + k0 / kBlk + c] = static_cast<uint8_t>(sc);
  }
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

// ============================================================================
// Hot path: persistent warp-specialised block-scaled MMA kernel
// ============================================================================
struct MmaParams {
  const uint8_t* Wq;  // weight tile images [E][NT][KT][16384]
  const uint8_t* Ws;  // weight scale images [E][NT][KT][1024]
  const uint16_t* x;  // bf16 [M, K] (fused prologue)
  const float* D;     // fp32 [E, K]
  const uint8_t* Aq;  // pre-quantised activation tile images [MT][KT][16384] (unfused)
  const uint8_t* As;  // their scale images [MT][KT][1024]
  uint16_t* y;        // bf16 [M, N]
  const int64_t* group_list;  // device [E] or nullptr (dense)
  int group_list_type;
  int E, M, N, K, NT, KT;
  int splits;          // split-K factor (1 = none)
  float* partial;      // [tilesMN][splits][128 * BT] fp32 when splits > 1
  uint32_t* counters;  // [tilesMN] arrival counters, zero between calls
  int32_t* status;     // optional device status word
};

template <int BT>
struct Cfg {
  static constexpr int kAccStride = BT < 32 ? 32 : BT;            // TMEM columns per accumulator
  static constexpr int kSfCol = 2 * kAccStride;                   // SFA at kSfCol, SFB at kSfCol + 8
  static constexpr int kTmemNeed = 2 * kAccStride + 16;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  static constexpr int kBBytes = BT * 128;                       // activation codes per stage
  static constexpr int kStageBytes = kTileCodeBytes + kBBytes + 2 * kTileSfBytes;
  static constexpr int kOffB = kTileCodeBytes;
  static constexpr int kOffSfa = kTileCodeBytes + kBBytes;
  static constexpr int kOffSfb = kOffSfa + kTileSfBytes;
  static constexpr int kBarOff = kStages * kStageBytes;           // barriers and small state
  static constexpr int kRbufOff = kBarOff + 256;                  // 2 x 256 fp32 reciprocals + 2 flags
  static constexpr int kScanOff = kRbufOff + 2 * kKTile * 4 + 64; // scan scratch (64 x int64)
  static constexpr int kGroupOff = kScanOff + 64 * 8;             // group tables
  static constexpr size_t smem_bytes(int E_grouped) {
    return 1024 + kGroupOff + (E_grouped > 0 ? static_cast<size_t>(E_grouped + 1) * 12 + 16 : 0);
  }
  static_assert(BT % 16 == 0 && BT >= 16 && BT <= 128, "token tile");
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
};

constexpr int kProWarps = 8;  // prologue warps (fused)
constexpr int kEpiWarp0 = 2;
constexpr int kProWarp0 = 6;
__host__ __device__ constexpr int mma_threads(bool fused) { return fused ? (kProWarp0 + kProWarps) * 32 : 192; }

struct TileInfo {
  int g, m0, rows, mg, nt, ks, kt0, kt1, mn;
};

// Block-wide exclusive scan of one int64 per thread (blockDim.x <= 1024).
__device__ __forceinline__ int64_t block_excl_scan(int64_t v, int64_t* scratch, int64_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
  int64_t inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t u = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += u;
  }
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int64_t w = lane < nw ? scratch[lane] : 0;
    int64_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int64_t u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    if (lane < nw) scratch[32 + lane] = wi - w;  // exclusive warp prefix
    if (lane == nw - 1) scratch[63] = wi;
  }
  __syncthreads();
  const int64_t res = scratch[32 + warp] + inc - v;
  total = scratch[63];
  __syncthreads();
  return res;
}

// Validates group_list on the device (npu_grouped_matmul rules) and builds
// row offsets goff[0..E] and m-tile prefix gtp[0..E].  Returns false if invalid.
template <int BT>
__device__ bool build_group_tables(const MmaParams& p, int64_t* goff, int* gtp, int64_t* scratch) {
  const int E = p.E;
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int g0 = threadIdx.x * per, g1 = min(E, g0 + per);
  int64_t cnt_sum = 0, tile_sum = 0;
  bool bad = false;
  for (int g = g0; g < g1; ++g) {
    const int64_t v = p.group_list[g];
    const int64_t prev = (p.group_list_type == 0 && g > 0) ? p.group_list[g - 1] : 0;
    const int64_t cnt = p.group_list_type == 0 ? v - prev : v;
    if (v < 0 || cnt < 0 || cnt > p.M) bad = true;
    cnt_sum += cnt;
    tile_sum += (cnt + BT - 1) / BT;
  }
  bad = __syncthreads_or(bad);
  if (bad) return false;
  int64_t rows_total, tiles_total;
  int64_t row_base = block_excl_scan(cnt_sum, scratch, rows_total);
  int64_t tile_base = block_excl_scan(tile_sum, scratch, tiles_total);
  if (rows_total != p.M) return false;  // uniform: every thread reads the same total
  for (int g = g0; g < g1; ++g) {
    const int64_t v = p.group_list[g];
    const int64_t prev = (p.group_list_type == 0 && g > 0) ? p.group_list[g - 1] : 0;
    const int64_t cnt = p.group_list_type == 0 ? v - prev : v;
    goff[g] = row_base;
    gtp[g] = static_cast<int>(tile_base);
    row_base += cnt;
    tile_base += (cnt + BT - 1) / BT;
  }
  if (threadIdx.x == 0) {
    goff[E] = rows_total;
    gtp[E] = static_cast<int>(tiles_total);
  }
  __syncthreads();
  return true;
}

template <int BT>
__device__ __forceinline__ TileInfo decode_tile(const MmaParams& p, int idx, const int64_t* goff, const int* gtp) {
  TileInfo ti;
  ti.ks = idx % p.splits;
  const int rest = idx / p.splits;
  ti.mn = rest;
  ti.nt = rest % p.NT;
  ti.mg = rest / p.NT;
  if (p.group_list == nullptr) {
    ti.g = 0;
    ti.m0 = ti.mg * BT;
    ti.rows = min(BT, p.M - ti.m0);
  } else {
    int lo = 0, hi = p.E;  // largest g with gtp[g] <= mg (skips empty groups)
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (gtp[mid] <= ti.mg) lo = mid; else hi = mid;
    }
    ti.g = lo;
    ti.m0 = static_cast<int>(goff[lo]) + (ti.mg - gtp[lo]) * BT;
    ti.rows = min(BT, static_cast<int>(goff[lo + 1]) - ti.m0);
  }
  ti.kt0 = static_cast<int>((static_cast<int64_t>(ti.ks) * p.KT) / p.splits);
  ti.kt1 = static_cast<int>((static_cast<int64_t>(ti.ks + 1) * p.KT) / p.splits);
  return ti;
}

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float v) {
  __nv_bfloat16 h = __float2bfloat16_rn(v);
  return *reinterpret_cast<uint16_t*>(&h);
}

template <int BT, bool kFused>
__global__ void __launch_bounds__(mma_threads(kFused), 1) mma_kernel(const __grid_constant__ MmaParams p) {
  using C = Cfg<BT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* acce = accf + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* epi_flag = abort_flag + 1;   // epilogue broadcast word
  volatile int* pro_flag = abort_flag + 2;   // prologue broadcast words [2]
  float* rbuf = reinterpret_cast<float*>(smem + C::kRbufOff);
  int64_t* scan_scratch = reinterpret_cast<int64_t*>(smem + C::kScanOff);
  int64_t* goff = reinterpret_cast<int64_t*>(smem + C::kGroupOff);
  int* gtp = reinterpret_cast<int*>(goff + (p.E + 1));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- tile space ----
  int total_mtiles;
  if (p.group_list != nullptr) {
    if (!build_group_tables<BT>(p, goff, gtp, scan_scratch)) {
      if (blockIdx.x == 0 && threadIdx.x == 0 && p.status) *p.status = MACAQ_ERR_GROUP_LIST_INVALID;
      return;
    }
    total_mtiles = gtp[p.E];
  } else {
    total_mtiles = ceil_div(p.M, BT);
  }
  const int total_tiles = total_mtiles * p.NT * p.splits;
  if (static_cast<int>(blockIdx.x) >= total_tiles) return;

  // ---- set-up ----
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], kFused ? 1 + kProWarps : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if constexpr (kFused) {
    // scale rows >= BT of the activation scale image are never written: zero them once
    for (int i = threadIdx.x; i < kStages * kTileSfBytes / 16; i += blockDim.x) {
      const int s = i / (kTileSfBytes / 16), o = i % (kTileSfBytes / 16);
      *reinterpret_cast<uint4*>(smem + s * C::kStageBytes + C::kOffSfb + o * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  if (warp == 0) {
    // ================= bulk-copy producer =================
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total_tiles && ok; idx += gridDim.x) {
        const TileInfo ti = decode_tile<BT>(p, idx, goff, gtp);
        for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitTimeoutNs)) { ok = false; break; }
          uint8_t* sb = smem + stage * C::kStageBytes;
          constexpr uint32_t bytes = kTileCodeBytes + kTileSfBytes + (kFused ? 0 : C::kBBytes + kTileSfBytes);
          mbar_arrive_expect_tx(&full[stage], bytes);
          const size_t wt = (static_cast<size_t>(ti.g) * p.NT + ti.nt) * p.KT + kt;
          bulk_g2s(sb, p.Wq + wt * kTileCodeBytes, kTileCodeBytes, &full[stage]);
          bulk_g2s(sb + C::kOffSfa, p.Ws + wt * kTileSfBytes, kTileSfBytes, &full[stage]);
          if constexpr (!kFused) {
            const size_t at = static_cast<size_t>(ti.mg) * p.KT + kt;
            bulk_g2s(sb + C::kOffB, p.Aq + at * kTileCodeBytes, C::kBBytes, &full[stage]);
            bulk_g2s(sb + C::kOffSfb, p.As + at * kTileSfBytes, kTileSfBytes, &full[stage]);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0) {
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      const uint32_t idesc_lo = idesc_mxf4(128, BT, 0, 0);
      const uint32_t idesc_hi = idesc_mxf4(128, BT, 2, 2);
      const uint32_t sfa_col = tmem + C::kSfCol, sfb_col = tmem + C::kSfCol + 8;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total_tiles && ok; idx += gridDim.x) {
        const TileInfo ti = decode_tile<BT>(p, idx, goff, gtp);
        if (!mbar_wait(&acce[acc], acc_phase ^ 1, abort_flag, kWaitTimeoutNs)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * C::kAccStride;
        for (int kt = ti.kt0; kt < ti.kt1; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag, kWaitTimeoutNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b_addr = a_addr + C::kOffB;
          const uint32_t sfa_addr = a_addr + C::kOffSfa, sfb_addr = a_addr + C::kOffSfb;
          tc_cp_32x128b_warpx4(sfa_col, sdesc_sf_block(sfa_addr));
          tc_cp_32x128b_warpx4(sfa_col + 4, sdesc_sf_block(sfa_addr + 512));
          tc_cp_32x128b_warpx4(sfb_col, sdesc_sf_block(sfb_addr));
          tc_cp_32x128b_warpx4(sfb_col + 4, sdesc_sf_block(sfb_addr + 512));
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint32_t sfid = static_cast<uint32_t>(k & 1) * 2u;
            const uint32_t sfa = (sfa_col + (k >> 1) * 4) | (sfid << 30);
            const uint32_t sfb = (sfb_col + (k >> 1) * 4) | (sfid << 30);
            tc_mma_mxf4(d_tmem, sdesc_kmajor_sw128(a_addr + 32 * k), sdesc_kmajor_sw128(b_addr + 32 * k),
                        (k & 1) ? idesc_hi : idesc_lo, sfa, sfb, (kt > ti.kt0 || k > 0) ? 1u : 0u);
          }
          tc_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        tc_commit(&accf[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
    }
  } else if (warp < kEpiWarp0 + 4) {
    // ================= epilogue =================
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int et = threadIdx.x - kEpiWarp0 * 32;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int idx = blockIdx.x; idx < total_tiles; idx += gridDim.x) {
      const TileInfo ti = decode_tile<BT>(p, idx, goff, gtp);
      if (et == 0) *epi_flag = mbar_wait(&accf[acc], acc_phase, abort_flag, kWaitTimeoutNs) ? 1 : 0;
      named_bar_sync(1, 128);
      if (!*epi_flag) break;
      tc_fence_after();
      const int n = ti.nt * kRowsTile + q * 32 + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccStride;
      if (p.splits == 1) {
#pragma unroll 1
        for (int c0 = 0; c0 < BT; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + c0, r);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int t = c0 + j;
              if (t < ti.rows)
                p.y[static_cast<int64_t>(ti.m0 + t) * p.N + n] = f32_to_bf16_bits(__uint_as_float(r[j]) * 0.03125f);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[acc]);
      } else {
        float* part = p.partial + (static_cast<size_t>(ti.mn) * p.splits + ti.ks) * (kRowsTile * BT);
#pragma unroll 1
        for (int c0 = 0; c0 < BT; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(taddr + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) __stcg(part + (c0 + j) * kRowsTile + q * 32 + lane, __uint_as_float(r[j]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acce[acc]);
        __threadfence();
        named_bar_sync(1, 128);
        if (et == 0) {
          const uint32_t old = atomicAdd(p.counters + ti.mn, 1u);
          *epi_flag = (old == static_cast<uint32_t>(p.splits - 1)) ? 2 : 1;
        }
        named_bar_sync(1, 128);
        if (*epi_flag == 2) {
          __threadfence();
          const float* base = p.partial + static_cast<size_t>(ti.mn) * p.splits * (kRowsTile * BT);
#pragma unroll 1
          for (int t = 0; t < ti.rows; ++t) {
            float s = 0.0f;
            for (int kk = 0; kk < p.splits; ++kk)
              s += __ldcg(base + static_cast<size_t>(kk) * (kRowsTile * BT) + t * kRowsTile + q * 32 + lane);
            if (n < p.N) p.y[static_cast<int64_t>(ti.m0 + t) * p.N + n] = f32_to_bf16_bits(s * 0.03125f);
          }
          if (et == 0) p.counters[ti.mn] = 0u;  // ready for the next call
        }
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  } else if constexpr (kFused) {
    // ================= activation prologue =================
    const int pt = threadIdx.x - kProWarp0 * 32;  // 0 .. 255
    constexpr int kPT = kProWarps * 32;
    int stage = 0, it = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < total_tiles && ok; idx += gridDim.x) {
      const TileInfo ti = decode_tile<BT>(p, idx, goff, gtp);
      const float* Dg = p.D + static_cast<size_t>(ti.g) * p.K;
      for (int kt = ti.kt0; kt < ti.kt1; ++kt, ++it) {
        float* r = rbuf + (it & 1) * kKTile;
        for (int j = pt; j < kKTile; j += kPT) r[j] = __frcp_rn(__ldg(Dg + kt * kKTile + j));
        if (pt == 0) pro_flag[it & 1] = mbar_wait(&empty[stage], phase ^ 1, abort_flag, kWaitTimeoutNs) ? 1 : 0;
        named_bar_sync(2, kPT);
        if (!pro_flag[it & 1]) { ok = false; break; }
        uint8_t* sb = smem + stage * C::kStageBytes;
        uint8_t* bcode = sb + C::kOffB;
        uint8_t* bsf = sb + C::kOffSfb;
#pragma unroll 1
        for (int task = pt; task < BT * 8; task += kPT) {
          const int t = task >> 3, c = task & 7;
          uint4 cv = make_uint4(0, 0, 0, 0);
          uint32_t sc = 0;
          if (t < ti.rows) {
            const uint4* src = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(ti.m0 + t) * p.K +
                                                              static_cast<int64_t>(kt) * kKTile + c * kBlk);
            uint4 xv[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) xv[i] = __ldg(src + i);
            act_block(xv, r + c * kBlk, cv, sc);
          }
          *reinterpret_cast<uint4*>(bcode + code_chunk_offset(t, c)) = cv;
          bsf[sf_offset(t, c)] = static_cast<uint8_t>(sc);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1; }
      }
    }
  }

  // ---- tear-down ----
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
};
DeviceState g_dev[kMaxDevices];

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
  return s.is_sm100 ? MACAQ_OK : MACAQ_ERR_ARCH;
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

// Smallest token tile that covers M (the swapped MMA's N dimension).
int pick_bt(int64_t rows_per_group) {
  if (rows_per_group <= 16) return 16;
  if (rows_per_group <= 32) return 32;
  if (rows_per_group <= 64) return 64;
  return 128;
}

// Split-K factor for a dense problem so that the grid covers the SMs.
int pick_splits(int64_t M, int64_t N, int64_t K, int bt, int sms) {
  const int64_t tiles = ((M + bt - 1) / bt) * ((N + 127) / 128);
  const int64_t KT = K / 256;
  if (tiles >= sms || tiles >= 1024) return 1;
  int64_t s = (sms + tiles - 1) / tiles;
  if (s > KT) s = KT;
  if (s > 32) s = 32;
  return static_cast<int>(s < 1 ? 1 : s);
}

// Split-K workspace: a fixed counter region first (so that its zeros survive
// calls of other shapes that reuse the same buffer), then the FP32 partials.
// Split-K is only chosen when the output tiles number fewer than the SMs.
constexpr size_t kCounterBytes = 4096;  // 1024 counters; pick_splits never splits 1024+ tiles

size_t dense_ws_bytes(int64_t M, int64_t N, int64_t K, int sms) {
  const int bt = pick_bt(M);
  const int s = pick_splits(M, N, K, bt, sms);
  if (s <= 1) return 0;
  const size_t tiles = static_cast<size_t>((M + bt - 1) / bt) * static_cast<size_t>((N + 127) / 128);
  return kCounterBytes + tiles * s * 128 * bt * sizeof(float);
}

template <int BT, bool F>
int launch_mma(const MmaParams& p, int grid, size_t smem, cudaStream_t st, int dev) {
  static bool attr_set[kMaxDevices] = {};
  static size_t attr_bytes[kMaxDevices] = {};
  if (!attr_set[dev] || attr_bytes[dev] < smem) {
    const size_t want = Cfg<BT>::smem_bytes(kMaxGroups);
    if (cudaFuncSetAttribute(mma_kernel<BT, F>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(want > smem ? want : smem)) != cudaSuccess)
      return MACAQ_ERR_CUDA;
    attr_set[dev] = true;
    attr_bytes[dev] = want > smem ? want : smem;
  }
  mma_kernel<BT, F><<<grid, mma_threads(F), smem, st>>>(p);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

int dispatch_mma(int bt, bool fused, const MmaParams& p, int grid, int E_grouped, cudaStream_t st, int dev) {
  switch (bt) {
    case 16:
      return launch_mma<16, true>(p, grid, Cfg<16>::smem_bytes(E_grouped), st, dev);
    case 32:
      return launch_mma<32, true>(p, grid, Cfg<32>::smem_bytes(E_grouped), st, dev);
    case 64:
      return launch_mma<64, true>(p, grid, Cfg<64>::smem_bytes(E_grouped), st, dev);
    default:
      if (fused) return launch_mma<128, true>(p, grid, Cfg<128>::smem_bytes(E_grouped), st, dev);
      return launch_mma<128, false>(p, grid, Cfg<128>::smem_bytes(E_grouped), st, dev);
  }
}

int check_dense_args(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y,
                     int64_t M, int64_t N, int64_t K, int64_t E) {
  if (M < 0 || M > INT32_MAX || !valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (M == 0) return MACAQ_OK;
  if (!x || !D || !Wq || !Ws || !y) return MACAQ_ERR_NULL;
  if (!aligned16(x) || !aligned16(D) || !aligned16(Wq) || !aligned16(Ws) || !aligned16(y)) return MACAQ_ERR_ALIGN;
  const size_t ybytes = static_cast<size_t>(M) * N * 2;
  if (overlaps(y, ybytes, x, static_cast<size_t>(M) * K * 2) || overlaps(y, ybytes, D, static_cast<size_t>(E) * K * 4) ||
      overlaps(y, ybytes, Wq, macaq_weight_code_bytes(E, N, K)) ||
      overlaps(y, ybytes, Ws, macaq_weight_scale_bytes(E, N, K)))
    return MACAQ_ERR_ALIAS;
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
    default: return "MACAQ_ERR_UNKNOWN";
  }
}

int macaq_abi_version(void) { return MACAQ_ABI_VERSION; }

size_t macaq_weight_code_bytes(int64_t E, int64_t N, int64_t K) {
  if (E < 1 || E > kMaxGroups || !valid_nk(N, K)) return 0;
  return static_cast<size_t>(E) * pad128(N) * (K / 2);
}

size_t macaq_weight_scale_bytes(int64_t E, int64_t N, int64_t K) {
  if (E < 1 || E > kMaxGroups || !valid_nk(N, K)) return 0;
  return static_cast<size_t>(E) * pad128(N) * (K / 32);
}

int macaq_prepare_weights(const float* W, const float* D, int64_t E, int64_t N, int64_t K, uint8_t* Wq, uint8_t* Ws,
                          void* stream) {
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (!valid_nk(N, K)) return MACAQ_ERR_SHAPE;
  if (!W || !D || !Wq || !Ws) return MACAQ_ERR_NULL;
  if (!aligned16(W) || !aligned16(D) || !aligned16(Wq) || !aligned16(Ws)) return MACAQ_ERR_ALIGN;
  const size_t qb = macaq_weight_code_bytes(E, N, K), sb = macaq_weight_scale_bytes(E, N, K);
  if (overlaps(Wq, qb, W, E * N * K * 4) || overlaps(Wq, qb, D, E * K * 4) || overlaps(Ws, sb, W, E * N * K * 4) ||
      overlaps(Ws, sb, D, E * K * 4) || overlaps(Wq, qb, Ws, sb))
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
  const int NT = static_cast<int>(pad128(N) / 128);
  dim3 grid(static_cast<unsigned>(E * NT * 4), static_cast<unsigned>(K / 256));
  prep_weights_kernel<<<grid, 256, 0, s>>>(W, D, Wq, Ws, static_cast<int>(N), static_cast<int>(K), NT);
  return cudaPeekAtLastError() == cudaSuccess ? MACAQ_OK : MACAQ_ERR_CUDA;
}

size_t macaq_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t E) {
  if (M <= 0 || !valid_nk(N, K) || E < 1 || E > kMaxGroups) return 0;
  if (E > 1) return 0;  // grouped calls run the fused kernel without split-K
  int dev, sms;
  if (current_device(dev, sms) != MACAQ_OK) sms = 148;
  return dense_ws_bytes(M, N, K, sms);
}

int macaq_dense_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y, int64_t M,
                   int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  int st = check_dense_args(x, D, Wq, Ws, y, M, N, K, 1);
  if (st != MACAQ_OK || M == 0) return st;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const int bt = pick_bt(M);
  const int splits = pick_splits(M, N, K, bt, sms);
  const size_t need = dense_ws_bytes(M, N, K, sms);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned16(workspace)))
    return MACAQ_ERR_WORKSPACE;
  MmaParams p{};
  p.Wq = Wq; p.Ws = Ws; p.x = x; p.D = D; p.y = y;
  p.group_list = nullptr; p.group_list_type = 0;
  p.E = 1; p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
  p.NT = static_cast<int>(pad128(N) / 128); p.KT = static_cast<int>(K / 256);
  p.splits = splits;
  p.status = status;
  if (splits > 1) {
    p.counters = static_cast<uint32_t*>(workspace);
    p.partial = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kCounterBytes);
  }
  const int64_t tiles_total = static_cast<int64_t>((M + bt - 1) / bt) * p.NT * splits;
  const int grid = static_cast<int>(tiles_total < sms ? tiles_total : sms);
  return dispatch_mma(bt, true, p, grid, 0, static_cast<cudaStream_t>(stream), dev);
}

int macaq_grouped_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws,
                     const int64_t* group_list, int group_list_type, int64_t E, uint16_t* y, int64_t M, int64_t N,
                     int64_t K, void* workspace, size_t workspace_bytes, int32_t* status, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (E < 1 || E > kMaxGroups) return MACAQ_ERR_TOO_MANY_GROUPS;
  if (group_list_type != 0 && group_list_type != 1) return MACAQ_ERR_GROUP_LIST_TYPE;
  int st = check_dense_args(x, D, Wq, Ws, y, M, N, K, E);
  if (st != MACAQ_OK) return st;
  if (M == 0) return MACAQ_OK;
  if (!group_list) return MACAQ_ERR_NULL;
  if (!aligned16(group_list)) return MACAQ_ERR_ALIGN;
  if (overlaps(y, static_cast<size_t>(M) * N * 2, group_list, E * 8)) return MACAQ_ERR_ALIAS;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const int bt = pick_bt((M + E - 1) / E);
  MmaParams p{};
  p.Wq = Wq; p.Ws = Ws; p.x = x; p.D = D; p.y = y;
  p.group_list = group_list; p.group_list_type = group_list_type;
  p.E = static_cast<int>(E); p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
  p.NT = static_cast<int>(pad128(N) / 128); p.KT = static_cast<int>(K / 256);
  p.splits = 1;
  p.status = status;
  return dispatch_mma(bt, true, p, sms, static_cast<int>(E), static_cast<cudaStream_t>(stream), dev);
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
  quant_act_kernel<false><<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, D, codes, scales, static_cast<int>(M), static_cast<int>(K), static_cast<int>(M));
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
      Wq, Ws, codes, scales, static_cast<int>(N), static_cast<int>(K), static_cast<int>(pad128(N) / 128),
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
  return static_cast<size_t>(pad128(M)) * (K / 2 + K / 32);
}

int macaq_unfused_dense_mm(const uint16_t* x, const float* D, const uint8_t* Wq, const uint8_t* Ws, uint16_t* y,
                           int64_t M, int64_t N, int64_t K, void* workspace, size_t workspace_bytes, int32_t* status,
                           void* stream) {
  int st = check_dense_args(x, D, Wq, Ws, y, M, N, K, 1);
  if (st != MACAQ_OK || M == 0) return st;
  int dev, sms;
  st = current_device(dev, sms);
  if (st != MACAQ_OK) return st;
  const size_t need = macaq_unfused_workspace_bytes(M, K);
  if (!workspace || workspace_bytes < need || !aligned16(workspace)) return MACAQ_ERR_WORKSPACE;
  if (overlaps(workspace, need, y, static_cast<size_t>(M) * N * 2)) return MACAQ_ERR_ALIAS;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t Mp = pad128(M);
  uint8_t* Aq = static_cast<uint8_t*>(workspace);
  uint8_t* As = Aq + static_cast<size_t>(Mp) * (K / 2);
  dim3 qgrid(static_cast<unsigned>(Mp / 32), static_cast<unsigned>(K / 256));
  quant_act_kernel<true><<<qgrid, 256, 0, s>>>(x, D, Aq, As, static_cast<int>(M), static_cast<int>(K),
                                                static_cast<int>(Mp));
  if (cudaPeekAtLastError() != cudaSuccess) return MACAQ_ERR_CUDA;
  MmaParams p{};
  p.Wq = Wq; p.Ws = Ws; p.Aq = Aq; p.As = As; p.D = D; p.y = y;
  p.E = 1; p.M = static_cast<int>(M); p.N = static_cast<int>(N); p.K = static_cast<int>(K);
  p.NT = static_cast<int>(pad128(N) / 128); p.KT = static_cast<int>(K / 256);
  p.splits = 1;
  p.status = status;
  const int64_t tiles = (Mp / 128) * p.NT;
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  return dispatch_mma(128, false, p, grid, 0, s, dev);
}

}  // extern "C"
