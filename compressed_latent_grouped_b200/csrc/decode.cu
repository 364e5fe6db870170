// Decode path: one new token per sequence against the latent KV cache
// ("Compressed Convolutional Attention", Probleemstelling 2: the KV cache grows
// with the sequence and decode is bound by reading it; Resultaten 3: the cache
// shrinks with C.  "Grouped Query Attention (GQA)", "Por qué GQA reduce la
// caché KV": decode speed is set by memory bandwidth).
//
//   kv_append        bit-exact copy of new rows into the cache at len[b]
//   decode_proj      x_t W^T for all sequences, split over E (fp32 partials)
//   decode_pre       one-token conv from the stored history, channel mix,
//                    QK-mean, RoPE at position len[b], value-shift from the
//                    stored previous row, cache append, state update
//   decode_attn      split-K attention over len[b] + 1 keys: each CTA streams
//                    one chunk of K and V of one kv group with bulk copies
//                    through a shared-memory ring; every K/V row read serves
//                    all G query heads.  The last CTA of a (sequence, group)
//                    -- found with an atomic ticket, never by waiting --
//                    merges the chunks; the last group of a sequence bumps len.
#include <cmath>

#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {

// ----------------------------------------------------------------- split plan
// Few sequences: the projection streams W once, one warp per output column,
// with x (B x E, working dtype) held in shared memory.
constexpr int kGvMaxB = 16;
constexpr size_t kGvMaxX = 64 * 1024;
static bool decode_use_gemv(int B, int E, int es) {
  // x fits in shared memory, and a W row is a whole number of 512-byte steps
  // (32 lanes x 16 bytes), at most 16 of them (held in registers)
  const size_t row = static_cast<size_t>(E) * es;
  return B <= kGvMaxB && static_cast<size_t>(B) * row <= kGvMaxX && row % 512 == 0 &&
         row <= 512 * 16;
}
// More sequences, bf16: the projection on the tensor core, swapped (W rows as M),
// one CTA per (128 W rows, 64 sequences, 128 of E).
// Tensor-core decode projection tiles: 128 W rows x 64 sequences x 128 of E
// (2 blocks of 64, both staged in one round of TMA).  Measured at 64 sequences,
// E = 4096: 512 of E per CTA (48 CTAs, a quarter of the partials) took 13.6 us
// against 12.8 us; the pre-step summing fewer partials gained under 1 us.
constexpr int kDpN = 128, kDpB = 64, kDpK = 128, kDpKB = kDpK / 64;
static bool decode_use_proj_tc(int E, int es) { return es == 2 && E % kDpK == 0; }

// E range of one projection split: E / e_splits rounded up to whole 64-wide steps.
static int decode_proj_e_len(int E, int e_splits) {
  const int per = (E + e_splits - 1) / e_splits;
  return (per + 63) / 64 * 64;
}

void decode_plan(int B, int Hkv, int E, int N, int64_t cap, bool has_proj, int es,
                 int* e_splits, int* splits, int* chunk) {
  const int sms = sm_count();
  const int target = 2 * sms;
  if (has_proj && decode_use_gemv(B, E, es)) {
    *e_splits = 1;   // one weight-streaming pass, no partials to sum
  } else if (has_proj && decode_use_proj_tc(E, es)) {
    *e_splits = E / kDpK;   // tensor-core tiles of 128 columns x 64 sequences x kDpK of E
  } else if (has_proj) {
    // projection CTAs: 64 columns x 64 sequences x one E-split of whole 64-wide steps
    const int tiles = ((N + 63) / 64) * ((B + 63) / 64);
    int nsp = target / (tiles > 0 ? tiles : 1);
    if (nsp < 1) nsp = 1;
    const int e_len = decode_proj_e_len(E, nsp);
    *e_splits = (E + e_len - 1) / e_len;
  } else {
    *e_splits = 0;
  }
  // Splits of whole 128-key chunks.  The CTAs of one launch should fill a whole
  // number of waves of the resident slots (SMs x 2 CTAs), each CTA
  // streaming at least ~1024 keys so its start-up cost stays small, and never
  // fewer than 4 chunks (512 keys) when the cache has that many: measured on
  // B200, a launch of a few hundred 2-chunk CTAs spends longer starting them
  // (about 37 per microsecond) and merging their partials than streaming keys.
  const int64_t bh = static_cast<int64_t>(B) * Hkv;
  const int64_t slots = static_cast<int64_t>(sms) * 2;
  const int64_t max_sp = (cap + 127) / 128;
  int64_t best_sp = 1;
  double best = -1.0;
  for (int64_t spc = 1; spc <= max_sp && spc <= 64; ++spc) {
    const int64_t chk = ((cap + spc - 1) / spc + 127) / 128 * 128;
    if (spc > 1 && chk < 512) break;   // fewer splits only from here on
    const int64_t real_sp = (cap + chk - 1) / chk;
    const int64_t ctas = bh * real_sp;
    const double waves = static_cast<double>(ctas) / slots;
    double eff = waves / std::ceil(waves);
    if (chk < 1024 && spc > 1) eff -= 0.25 * (1024 - chk) / 1024.0;
    if (eff > best + 1e-9) {
      best = eff;
      best_sp = real_sp;
    }
  }
  int64_t sp = best_sp;
  int64_t ch = (cap + sp - 1) / sp;
  ch = (ch + 127) / 128 * 128;
  *chunk = static_cast<int>(ch);
  *splits = static_cast<int>((cap + ch - 1) / ch);
}

namespace {

using namespace sm100;

// ----------------------------------------------------------------- kv append
// Rows i in [0, n) of sequence b go to token t0 + i, t0 = len[b] (append) or
// 0 (scatter); the source row of (b, i, g) is b sb + i si + g sg.
template <typename T>
__global__ void kv_append_kernel(T* __restrict__ ck, T* __restrict__ cv, const PageMap pm,
                                 const int32_t* len, const T* __restrict__ kn,
                                 const T* __restrict__ vn, int64_t sb, int64_t si, int64_t sg,
                                 int Hkv, int d, int64_t cap, int n_new, int32_t* dev_err) {
  constexpr int VEC = 16 / sizeof(T);
  const int b = blockIdx.y;
  const int L = len ? len[b] : 0;
  if (L < 0 || static_cast<int64_t>(L) + n_new > cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) raise_dev_err(dev_err, CCGQA_DEVERR_CAPACITY);
    return;
  }
  const int nch = d / VEC;
  const int64_t total = static_cast<int64_t>(n_new) * Hkv * nch;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = static_cast<int>(idx % nch);
    const int64_t rg = idx / nch;
    const int g = static_cast<int>(rg % Hkv);
    const int64_t i = rg / Hkv;
    const int64_t src = (b * sb + i * si + g * sg) * d + c * VEC;
    const int64_t row = kv_row(pm, b, g, Hkv, cap, L + i);
    if (row < 0) {
      raise_dev_err(dev_err, CCGQA_DEVERR_INDEX);
      continue;
    }
    const int64_t dst = row * d + c * VEC;
    *reinterpret_cast<uint4*>(ck + dst) = *reinterpret_cast<const uint4*>(kn + src);
    *reinterpret_cast<uint4*>(cv + dst) = *reinterpret_cast<const uint4*>(vn + src);
  }
}

__global__ void len_add_kernel(int32_t* len, int B, int64_t cap, int n_new) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B && len[b] >= 0 && static_cast<int64_t>(len[b]) + n_new <= cap) len[b] += n_new;
}

// ----------------------------------------------------------------- projection
// part[s][b][n] = sum over k in split s of x[b][k] W[n][k]: one CTA per (64
// columns, E-split, 64 sequences); both operands staged through shared memory
// with 16-byte loads, a 4 x 4 register tile per thread, float4 partial stores.
constexpr int kPB = 64, kPN = 64, kPK = 64;

template <typename T>
__device__ __forceinline__ void load16(const T* p, float (&v)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 2) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  } else {
    const float4 r = *reinterpret_cast<const float4*>(p);
    v[0] = r.x;
    v[1] = r.y;
    v[2] = r.z;
    v[3] = r.w;
  }
}

template <typename T>
__global__ void __launch_bounds__(256)
    decode_proj_kernel(const T* __restrict__ x, const T* __restrict__ W, float* __restrict__ part,
                       int B, int E, int N, int e_len) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int CPR = kPK / VEC;          // 16-byte chunks per staged row
  __shared__ __align__(16) float xs[kPK][kPB + 4];   // [k][sequence]
  __shared__ __align__(16) float wsm[kPK][kPN + 4];  // [k][column]
  const int n0 = blockIdx.x * kPN, sp = blockIdx.y, b0 = blockIdx.z * kPB;
  const int e_lo = sp * e_len, e_hi = min(E, e_lo + e_len);
  const int tb = threadIdx.x / 16, tn = threadIdx.x % 16;
  float acc[4][4] = {};
  for (int e0 = e_lo; e0 < e_hi; e0 += kPK) {
    // lanes run over rows, so the transposed shared-memory stores do not conflict
    for (int idx = threadIdx.x; idx < kPB * CPR; idx += 256) {
      const int r = idx % kPB, c = idx / kPB;
      const int gb = b0 + r, ge = e0 + c * VEC;
      float v[VEC];
      if (gb < B && ge < e_hi) {
        load16(x + static_cast<int64_t>(gb) * E + ge, v);
      } else {
#pragma unroll
        for (int u = 0; u < VEC; ++u) v[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < VEC; ++u) xs[c * VEC + u][r] = v[u];
    }
    for (int idx = threadIdx.x; idx < kPN * CPR; idx += 256) {
      const int r = idx % kPN, c = idx / kPN;
      const int gn = n0 + r, ge = e0 + c * VEC;
      float v[VEC];
      if (gn < N && ge < e_hi) {
        load16(W + static_cast<int64_t>(gn) * E + ge, v);
      } else {
#pragma unroll
        for (int u = 0; u < VEC; ++u) v[u] = 0.f;
      }
#pragma unroll
      for (int u = 0; u < VEC; ++u) wsm[c * VEC + u][r] = v[u];
    }
    __syncthreads();
#pragma unroll 16
    for (int k = 0; k < kPK; ++k) {
      const float4 xv = *reinterpret_cast<const float4*>(&xs[k][tb * 4]);
      const float4 wv = *reinterpret_cast<const float4*>(&wsm[k][tn * 4]);
      const float xr[4] = {xv.x, xv.y, xv.z, xv.w};
      const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(xr[i], wr[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gb = b0 + tb * 4 + i;
    if (gb >= B) continue;
    const int gn = n0 + tn * 4;
    float* dst = part + (static_cast<int64_t>(sp) * B + gb) * N + gn;
    if (gn + 3 < N && (N & 3) == 0) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (gn + j < N) dst[j] = acc[i][j];
    }
  }
}

// out[b][n] = sum_k x[b][k] W[n][k] for B <= BB (<= 16): one warp per output
// column.  A warp first issues every 16-byte load of its W row (the row stays
// in registers as raw 16-byte words), then the CTA stages x in shared memory,
// so the two memory latencies overlap; the products are reduced across lanes.
constexpr int kGvMaxIt = 16;   // 16-byte words per lane: E <= 32 * kGvMaxIt * (16 / sizeof(T))

template <typename T, int BB>
__global__ void __launch_bounds__(256)
    decode_gemv_kernel(const T* __restrict__ x, const T* __restrict__ W, float* __restrict__ out,
                       int B, int E, int N) {
  pdl_enter();
  constexpr int VEC = 16 / sizeof(T);
  extern __shared__ float4 gv_f4[];
  T* xs = reinterpret_cast<T*>(gv_f4);             // [B][E]
  const int lane = threadIdx.x & 31;
  const int n = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int nit = E / (32 * VEC);
  uint4 wraw[kGvMaxIt];
  if (n < N) {
    const uint4* wr = reinterpret_cast<const uint4*>(W + static_cast<int64_t>(n) * E) + lane;
#pragma unroll
    for (int it = 0; it < kGvMaxIt; ++it)
      if (it < nit) wraw[it] = __ldg(wr + it * 32);
  }
#pragma unroll 4
  for (int idx = threadIdx.x; idx < B * E / VEC; idx += blockDim.x)
    reinterpret_cast<uint4*>(xs)[idx] = reinterpret_cast<const uint4*>(x)[idx];
  __syncthreads();
  if (n >= N) return;
  float acc[BB];
#pragma unroll
  for (int b = 0; b < BB; ++b) acc[b] = 0.f;
#pragma unroll
  for (int it = 0; it < kGvMaxIt; ++it) {
    if (it >= nit) break;
    float wv[VEC];
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&wraw[it]);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        wv[2 * i] = f.x;
        wv[2 * i + 1] = f.y;
      }
    } else {
      const float4 f = *reinterpret_cast<const float4*>(&wraw[it]);
      wv[0] = f.x;
      wv[1] = f.y;
      wv[2] = f.z;
      wv[3] = f.w;
    }
    const int k0 = (it * 32 + lane) * VEC;
#pragma unroll
    for (int b = 0; b < BB; ++b) {
      if (b < B) {
        float xv[VEC];
        load16(xs + b * E + k0, xv);
#pragma unroll
        for (int u = 0; u < VEC; ++u) acc[b] = fmaf(wv[u], xv[u], acc[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < BB; ++b) {
    if (b < B) {
      float v = acc[b];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0) out[static_cast<int64_t>(b) * N + n] = v;
    }
  }
}

template <typename T>
cudaError_t launch_gemv(const T* x, const T* W, float* out, int B, int E, int N,
                        cudaStream_t stream) {
  const size_t xb = static_cast<size_t>(B) * E * sizeof(T);
  const int blocks = (N + 7) / 8;   // one warp per column
  auto go = [&](auto kernel) -> cudaError_t {
    if (xb > 48 * 1024) {
      cudaError_t e = allow_smem(reinterpret_cast<const void*>(kernel), static_cast<int>(xb));
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(kernel, dim3(blocks), dim3(256), xb, stream, x, W, out, B, E, N);
  };
  if (B <= 1) return go(decode_gemv_kernel<T, 1>);
  if (B <= 2) return go(decode_gemv_kernel<T, 2>);
  if (B <= 4) return go(decode_gemv_kernel<T, 4>);
  if (B <= 8) return go(decode_gemv_kernel<T, 8>);
  return go(decode_gemv_kernel<T, 16>);
}

// part[s][b][n] = sum over k in [kDpK s, kDpK (s + 1)) of W[n][k] x[b][k] on
// the tensor core: D^T = W_tile x_tile^T with M = 128 W rows, N = 64 sequences
// (rows past B read as zero), K = kDpK in steps of 16.  All 64-wide blocks of
// both tiles arrive by TMA in one round (128B swizzle), so a CTA costs one
// memory latency; one thread issues the MMAs; four warps read the accumulator
// back (lane = W row) and store fp32 partials, lanes over columns.
constexpr uint32_t kDpATile = kDpN * 64 * 2, kDpBTile = kDpB * 64 * 2;
constexpr size_t kDpSmem = kDpKB * (kDpATile + kDpBTile) + 64 + 1024;

__global__ void __launch_bounds__(128)
    decode_proj_tc_kernel(const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmX, float* __restrict__ part, int B,
                          int N, int32_t* dev_err) {
  pdl_enter();
  extern __shared__ uint8_t dp_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dp_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sa = smem;                          // [kDpKB][128 x 64] W blocks
  uint8_t* sb = smem + kDpKB * kDpATile;       // [kDpKB][64 x 64] x blocks
  uint64_t* full = reinterpret_cast<uint64_t*>(sb + kDpKB * kDpBTile);
  uint64_t* done = full + 1;
  uint64_t* drain = done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n0 = blockIdx.x * kDpN, sp = blockIdx.y, b0 = blockIdx.z * kDpB;
  const int e0 = sp * kDpK;
  if (tid == 0) {
    mbar_init(full, 1);
    mbar_init(done, 1);
    mbar_init(drain, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kDpB);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (tid == 0) {
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
    mbar_arrive_expect_tx(full, kDpKB * (kDpATile + kDpBTile));
#pragma unroll
    for (int kb = 0; kb < kDpKB; ++kb) {
      tma_load_2d(sa + kb * kDpATile, &tmW, full, e0 + kb * 64, n0);
      tma_load_2d(sb + kb * kDpBTile, &tmX, full, e0 + kb * 64, b0);
    }
    if (mbar_wait(full, 0, &abort_flag, dev_err)) {
      tc_fence_after();
      const uint32_t idesc = make_idesc_bf16(kDpN, kDpB, false);
#pragma unroll
      for (int kb = 0; kb < kDpKB; ++kb)
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t ad = make_smem_desc(smem_addr(sa + kb * kDpATile) + k * 32, 16, 1024,
                                             kSwizzle128B);
          const uint64_t bd = make_smem_desc(smem_addr(sb + kb * kDpBTile) + k * 32, 16, 1024,
                                             kSwizzle128B);
          mma_ss(tmem, ad, bd, idesc, (kb | k) != 0);
        }
      mma_commit(done);
    }
  }
  if (mbar_wait(done, 0, &abort_flag, dev_err)) {
    tc_fence_after();
    const uint32_t trow = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    uint32_t v0[32], v1[32];
    tmem_ld32(trow, v0);
    tmem_ld32(trow + 32, v1);
    tmem_wait_ld();
    const int n = n0 + warp * 32 + lane;
    if (n < N) {
#pragma unroll
      for (int c = 0; c < kDpB; ++c) {
        const int b = b0 + c;
        if (b < B)
          part[(static_cast<int64_t>(sp) * B + b) * N + n] = __uint_as_float(c < 32 ? v0[c] : v1[c - 32]);
      }
    }
  }
  if (abort_flag && tid == 0) {
    // Do not release TMEM while an MMA might still write it.
    mma_commit(drain);
    const long long c0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - c0 < kWaitLimitCycles) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kDpB);
  }
}

cudaError_t launch_decode_proj_tc(const bf16* x, const bf16* W, float* part, int B, int E, int N,
                                  int32_t* dev_err, cudaStream_t stream) {
  CUtensorMap tmW, tmX;
  const uint64_t dW[2] = {static_cast<uint64_t>(E), static_cast<uint64_t>(N)};
  const uint64_t dX[2] = {static_cast<uint64_t>(E), static_cast<uint64_t>(B)};
  const uint64_t st[1] = {static_cast<uint64_t>(E) * 2};
  const uint32_t bW[2] = {64, kDpN}, bX[2] = {64, kDpB};
  if (!encode_tensor_map(&tmW, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dW, st, bW,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tensor_map(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, dX, st, bX,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(decode_proj_tc_kernel),
                             static_cast<int>(kDpSmem));
  if (e != cudaSuccess) return e;
  dim3 grid((N + kDpN - 1) / kDpN, E / kDpK, (B + kDpB - 1) / kDpB);
  return launch_pdl(decode_proj_tc_kernel, grid, dim3(128), kDpSmem, stream, tmW, tmX, part, B,
                    N, dev_err);
}

// ----------------------------------------------------------------- pre-step

// Shared memory of the pre-step (byte offsets, each 16-byte aligned): fp32
// rows (current pre-conv row zc[AC], conv out u[HC], mix out y[HC], taps
// tp[HC][4]), the history rows hz[KH][HC] and the raw taps in the working
// dtype, and -- when they fit -- the group's G + 1 channel-mix weights, raw
// (as copied) and transposed.
struct PreSmem {
  size_t zc, u, y, tp, hz, tr, wt, wraw, bytes_no_w, bytes;
};
template <typename T>
__host__ __device__ inline PreSmem pre_smem(int G, int d, int K) {
  const int KH = K > 0 ? K - 1 : 0, HC = (G + 1) * d, AC = HC + d;
  auto up = [](size_t x) { return (x + 15) & ~size_t(15); };
  PreSmem L;
  L.zc = 0;
  L.u = up(L.zc + AC * 4);
  L.y = up(L.u + HC * 4);
  L.tp = up(L.y + HC * 4);
  L.hz = up(L.tp + HC * 16);
  L.tr = up(L.hz + static_cast<size_t>(KH) * HC * sizeof(T));
  L.wt = up(L.tr + static_cast<size_t>(HC) * (K > 0 ? K : 1) * sizeof(T));
  L.bytes_no_w = L.wt;
  const size_t wb = static_cast<size_t>(G + 1) * d * d * sizeof(T);
  L.wraw = up(L.wt + wb);
  L.bytes = up(L.wraw + wb);
  return L;
}
constexpr size_t kPreSmemMax = 200 * 1024;
// One CTA per (sequence, kv group); its work is a handful of dependent phases,
// each limited by one round of global loads, so every loop below is unrolled
// to keep several independent loads in flight per thread.
constexpr int kPreThreads = 256;

template <typename T>
__global__ void __launch_bounds__(kPreThreads) decode_pre_kernel(const __grid_constant__ DecodeArgs<T> a,
                                                         int stage_wt) {
  pdl_enter();
  extern __shared__ float4 dsm_f4[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(dsm_f4);
  const int g = blockIdx.x, b = blockIdx.y;
  const int d = a.d, G = a.G, K = a.K, half = d / 2;
  const int KH = K > 0 ? K - 1 : 0;
  const int QC = G * d, HC = QC + d, AC = HC + d;  // q | k | v channels of the group
  const PreSmem Ls = pre_smem<T>(G, d, K);
  float* zc = reinterpret_cast<float*>(sm + Ls.zc);   // [AC] current pre-conv row
  float* u = reinterpret_cast<float*>(sm + Ls.u);     // [HC]
  float* y = reinterpret_cast<float*>(sm + Ls.y);     // [HC]
  float* tp = reinterpret_cast<float*>(sm + Ls.tp);   // [HC][4] conv taps, zero past K
  T* hz = reinterpret_cast<T*>(sm + Ls.hz);           // [KH][HC] history rows
  T* tr = reinterpret_cast<T*>(sm + Ls.tr);           // [HC][K] taps as stored
  T* wt = reinterpret_cast<T*>(sm + Ls.wt);           // [G+1][d][d] mix weights, transposed
  T* wraw = reinterpret_cast<T*>(sm + Ls.wraw);       // [G+1][d][d] mix weights, as stored
  const int tid = threadIdx.x;
  const int L = __ldcg(a.len + b);
  if (L < 0 || L >= a.cap) {
    if (g == 0 && tid == 0) raise_dev_err(a.dev_err, CCGQA_DEVERR_CAPACITY);
    return;
  }
  // Paged cache: bring the sequence's block-table entries for tokens 0..L into
  // L2, so that the attention's CTAs find their page ids there when they start.
  if (a.pages.table != nullptr && g == 0) {
    const int32_t* row = a.pages.table + static_cast<int64_t>(b) * a.pages.per_seq;
    const int last = L >> a.pages.shift;
    for (int i = tid * 32; i <= last; i += blockDim.x * 32) prefetch_l2(row + i);
    if (tid == 0) prefetch_l2(row + last);   // the row need not start on a line
  }
  const int qcol0 = g * G * d, kcol0 = a.Hq * d + g * d, vcol0 = (a.Hq + a.Hkv) * d + g * d;
  // temporal channel conv: per-tap d x d matrices (wq_chan [Hq, K, d, d]), no depthwise taps
  const bool full = a.channel_conv && K > 0;
  const bool have_mix = K > 0 && !full && a.wq_chan != nullptr && a.wk_chan != nullptr;
  // 1. every input in one round of memory latency: the weights, taps and
  // history rows by 16-byte cp.async (contiguous per group), the projection
  // partials summed meanwhile
  {
    constexpr int VEC = 16 / sizeof(T);
    auto copy = [&](T* dst, const T* src, int n) {   // n elements, a multiple of VEC
      for (int i = tid * VEC; i < n; i += blockDim.x * VEC) cp_async16(dst + i, src + i);
    };
    if (stage_wt && have_mix) {
      copy(wraw, a.wq_chan + static_cast<int64_t>(g) * G * d * d, G * d * d);
      copy(wraw + G * d * d, a.wk_chan + static_cast<int64_t>(g) * d * d, d * d);
    }
    if (K > 0 && !full) {
      copy(tr, a.wq_seq + static_cast<int64_t>(g) * G * d * K, G * d * K);
      copy(tr + G * d * K, a.wk_seq + static_cast<int64_t>(g) * d * K, d * K);
    }
    for (int r = 0; r < KH; ++r) {
      copy(hz + r * HC, a.hist_q + (static_cast<int64_t>(b) * KH + r) * a.Hq * d + qcol0, QC);
      copy(hz + r * HC + QC, a.hist_k + (static_cast<int64_t>(b) * KH + r) * a.Hkv * d + g * d, d);
    }
    cp_async_commit_group();
  }
#pragma unroll 2
  for (int c = tid; c < AC; c += blockDim.x) {
    const int col = c < QC ? qcol0 + c : (c < HC ? kcol0 + (c - QC) : vcol0 + (c - HC));
    float val;
    if (a.W) {
      val = 0.f;
      const float* pp = a.proj_part + static_cast<int64_t>(b) * a.N + col;
      const int64_t pstride = static_cast<int64_t>(a.B) * a.N;
      // all partials loaded first, then summed in split order (deterministic)
      float pv[8];
      int s = 0;
      for (; s + 8 <= a.e_splits; s += 8) {
#pragma unroll
        for (int q = 0; q < 8; ++q) pv[q] = __ldcg(pp + (s + q) * pstride);
#pragma unroll
        for (int q = 0; q < 8; ++q) val += pv[q];
      }
      for (; s < a.e_splits; ++s) val += __ldcg(pp + s * pstride);
      val = to_f32(from_f32<T>(val));  // the projection output is held in the working dtype
    } else {
      val = to_f32(a.x_t[static_cast<int64_t>(b) * a.N + col]);
    }
    zc[c] = val;
  }
  cp_async_wait_all_groups();
  __syncthreads();
  // 2. shared-memory reshuffles: taps to fp32 [HC][4]; mix weights transposed,
  // wt[hh][j][i] = W_hh[i][j] (lanes run over rows i: consecutive stores)
  for (int idx = tid; !full && idx < HC * 4; idx += blockDim.x) {
    const int c = idx >> 2, j = idx & 3;
    tp[idx] = j < K ? to_f32(tr[c * K + j]) : 0.f;
  }
  if (stage_wt && have_mix) {
    // 16-byte words of W rows out, scattered into columns (lanes over rows i)
    constexpr int VEC = 16 / sizeof(T);
    const int per_head = d * d / VEC;
    for (int idx = tid; idx < (G + 1) * per_head; idx += blockDim.x) {
      const int hh = idx / per_head, rem = idx - hh * per_head;
      const int i = rem % d, j0 = (rem / d) * VEC;
      T v[VEC];
      *reinterpret_cast<uint4*>(v) = *reinterpret_cast<const uint4*>(wraw + (hh * d + i) * d + j0);
#pragma unroll
      for (int q = 0; q < VEC; ++q) wt[(hh * d + j0 + q) * d + i] = v[q];
    }
  }
  __syncthreads();
  // causal conv: tap j reads the row j steps back (history row KH - j)
  for (int c = tid; c < HC; c += blockDim.x) {
    float acc;
    if (K > 0 && !full) {
      const float* w = tp + c * 4;
      acc = w[0] * zc[c];
      for (int j = 1; j < K; ++j) acc = fmaf(w[j], to_f32(hz[(KH - j) * HC + c]), acc);
    } else {
      acc = zc[c];
    }
    u[c] = acc;
  }
  __syncthreads();
  // channel mix + QK-mean
  for (int c = tid; c < HC; c += blockDim.x) {
    const bool is_q = c < QC;
    const int hh = c / d, i = c - hh * d;
    const T* wch = is_q ? a.wq_chan : a.wk_chan;
    float acc;
    if (full) {
      // y[i] = sum_k sum_j W_k[i][j] z[t - k, j]; row t - k is history row KH - k
      const int head = is_q ? g * G + hh : g;
      const T* wh = wch + static_cast<int64_t>(head) * K * d * d + static_cast<int64_t>(i) * d;
      acc = 0.f;
      for (int k = 0; k < K; ++k) {
        const T* wr = wh + static_cast<int64_t>(k) * d * d;
        if (k == 0) {
#pragma unroll 8
          for (int j = 0; j < d; ++j) acc = fmaf(to_f32(wr[j]), zc[hh * d + j], acc);
        } else {
          const T* zr = hz + (KH - k) * HC + hh * d;
#pragma unroll 8
          for (int j = 0; j < d; ++j) acc = fmaf(to_f32(wr[j]), to_f32(zr[j]), acc);
        }
      }
    } else if (K > 0 && wch && stage_wt && have_mix) {
      const T* wc = wt + static_cast<int64_t>(hh) * d * d + i;   // column i of W_hh^T
      acc = 0.f;
#pragma unroll 8
      for (int j = 0; j < d; ++j) acc = fmaf(to_f32(wc[j * d]), u[hh * d + j], acc);
    } else if (K > 0 && wch) {
      const int head = is_q ? g * G + hh : g;
      const T* wr = wch + (static_cast<int64_t>(head) * d + i) * d;
      acc = 0.f;
      for (int j = 0; j < d; ++j) acc = fmaf(to_f32(wr[j]), u[hh * d + j], acc);
    } else {
      acc = u[c];
    }
    if (a.qk_mean == 2) {
      acc = 0.5f * (acc + zc[c]);   // "self": the head's own pre-conv value
    } else if (a.qk_mean) {
      float qp;
      if (is_q) {
        qp = zc[c];
      } else {
        qp = 0.f;
        for (int hl = 0; hl < G; ++hl) qp += zc[hl * d + i];
        qp /= static_cast<float>(G);
      }
      acc += 0.5f * (qp + zc[QC + i]);
    }
    y[c] = acc;
  }
  __syncthreads();
  // RoPE at position L on (i, i + d/2), then q -> workspace, k -> cache row L
  // (a page id outside the pool: the cache row is not written)
  const int64_t crow_i = kv_row(a.pages, b, g, a.Hkv, a.cap, L);
  const int64_t crow = crow_i * d;
  if (crow_i < 0 && tid == 0) raise_dev_err(a.dev_err, CCGQA_DEVERR_INDEX);
  for (int idx = tid; idx < (G + 1) * half; idx += blockDim.x) {
    const int hh = idx / half, i = idx - hh * half;
    float ya = y[hh * d + i], yb = y[hh * d + i + half];
    if (a.rope_on) {
      // angle L * theta_i reduced modulo one turn exactly in 64-bit fixed point
      const uint64_t ph = static_cast<uint64_t>(L) * a.rope_frac[i];
      const float f = static_cast<float>(static_cast<int64_t>(ph)) * 5.42101086242752217e-20f;
      float s, c;
      sincospif(2.0f * f, &s, &c);
      const float na = ya * c - yb * s, nb = ya * s + yb * c;
      ya = na;
      yb = nb;
    }
    if (hh < G) {
      float* qd = a.q_ws + (static_cast<int64_t>(b) * a.Hq + g * G + hh) * d;
      qd[i] = ya;
      qd[i + half] = yb;
    } else if (crow_i >= 0) {
      a.cache_k[crow + i] = from_f32<T>(ya);
      a.cache_k[crow + i + half] = from_f32<T>(yb);
    }
  }
  const bool shift_head = a.value_shift == 2 && g >= a.Hkv - a.Hkv / 2;
  for (int i = tid; i < d; i += blockDim.x) {
    T v = from_f32<T>(zc[HC + i]);
    if ((a.value_shift == 1 && i >= half) || shift_head)
      v = a.v_prev[static_cast<int64_t>(b) * a.Hkv * d + g * d + i];
    if (crow_i >= 0) a.cache_v[crow + i] = v;
  }
  __syncthreads();
  // state: histories shift by one row, v_prev = this row's v~
  for (int idx = tid; idx < KH * HC; idx += blockDim.x) {
    const int r = idx / HC, c = idx - r * HC;
    const float val = (r + 1 < KH) ? to_f32(hz[(r + 1) * HC + c]) : zc[c];
    if (c < QC)
      a.hist_q[(static_cast<int64_t>(b) * KH + r) * a.Hq * d + qcol0 + c] = from_f32<T>(val);
    else
      a.hist_k[(static_cast<int64_t>(b) * KH + r) * a.Hkv * d + g * d + (c - QC)] = from_f32<T>(val);
  }
  if (a.v_prev) {
    for (int i = tid; i < d; i += blockDim.x)
      a.v_prev[static_cast<int64_t>(b) * a.Hkv * d + g * d + i] = from_f32<T>(zc[HC + i]);
  }
}

// ----------------------------------------------------------------- attention
constexpr int kDecThreads = 128, kDecStages = 4, kPPMax = 4;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename T, int D>
struct DecCfg {
  static constexpr int CH = 16 / sizeof(T);  // elements per 16-byte chunk
  static constexpr int NCH = D / CH;         // chunks per row
  static constexpr int KS_raw = 8192 / (D * static_cast<int>(sizeof(T)));
  static constexpr int KS = KS_raw > 64 ? 64 : (KS_raw < 16 ? 16 : KS_raw);  // keys per stage
  static constexpr int KW = KS / 4;          // keys per warp per stage
  static constexpr uint32_t kStageBytes = 2u * KS * D * sizeof(T);
};

// CTAs per (split, kv group): each takes at most 32 kPPMax (head, chunk) pairs.
template <typename T, int D>
__host__ __device__ inline int dec_head_chunks(int G) {
  constexpr int per = 32 * kPPMax / DecCfg<T, D>::NCH;   // heads per CTA
  return (G + per - 1) / per;
}

// One stage of a paged cache: one bulk copy per run of rows within a page (the
// bytes are counted in a first pass); a page id outside the pool is not loaded
// (its rows keep what the stage held) and raises the index bit.  Kept out of
// line: only the issuing thread runs it.
template <typename T, int D>
__device__ __noinline__ void issue_paged_rows(const PageMap pm, const T* ck, const T* cv, int Hkv,
                                              int64_t cap, int32_t* dev_err, int b, int g,
                                              int key0, int rows, uint8_t* dst_k, uint8_t* dst_v,
                                              uint64_t* bar) {
  const int psz = 1 << pm.shift;
  uint32_t tx = 0;
  for (int r = 0; r < rows;) {
    const int t = key0 + r;
    const int run = min(rows - r, psz - (t & (psz - 1)));
    if (kv_row(pm, b, g, Hkv, cap, t) >= 0)
      tx += 2u * static_cast<uint32_t>(run) * D * sizeof(T);
    else
      raise_dev_err(dev_err, CCGQA_DEVERR_INDEX);
    r += run;
  }
  mbar_arrive_expect_tx(bar, tx);
  for (int r = 0; r < rows;) {
    const int t = key0 + r;
    const int run = min(rows - r, psz - (t & (psz - 1)));
    const int64_t row = kv_row(pm, b, g, Hkv, cap, t);
    if (row >= 0) {
      const uint32_t nb = static_cast<uint32_t>(run) * D * sizeof(T);
      bulk_load(dst_k + r * D * sizeof(T), ck + row * D, nb, bar);
      bulk_load(dst_v + r * D * sizeof(T), cv + row * D, nb, bar);
    }
    r += run;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads)
    decode_attn_kernel(const DecodeArgs<T> a) {
  using C = DecCfg<T, D>;
  extern __shared__ uint8_t dsm_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsm_raw) + 127) & ~uintptr_t(127));
  uint64_t* full = reinterpret_cast<uint64_t*>(ring + kDecStages * C::kStageBytes);
  float* wbuf = reinterpret_cast<float*>(full + kDecStages);  // merge scratch
  __shared__ int abort_flag, last_flag;

  // blockIdx.y = kv group x head chunk: a CTA serves at most 32 kPPMax / NCH
  // of the group's G query heads (heads hc0 .. hc0 + Gc - 1)
  const int n_hc = dec_head_chunks<T, D>(a.G);
  const int sp = blockIdx.x, g = blockIdx.y / n_hc, hc = blockIdx.y % n_hc, b = blockIdx.z;
  const int G = a.G, Gmax = (G + n_hc - 1) / n_hc, hc0 = hc * Gmax;
  const int Gc = min(Gmax, G - hc0), P = Gc * C::NCH;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int L = __ldcg(a.len + b);
  const bool valid_b = L >= 0 && L < a.cap;
  const int n_keys = valid_b ? L + 1 : 0;
  const int k0 = sp * a.chunk;
  const int k1 = min(k0 + a.chunk, n_keys);
  const int nk = max(0, k1 - k0);
  const int n_st = (nk + C::KS - 1) / C::KS;

  if (tid == 0) {
    for (int s = 0; s < kDecStages; ++s) mbar_init(&full[s], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  auto issue = [&](int st_idx) {
    const int s = st_idx % kDecStages;
    const int key0 = k0 + st_idx * C::KS;
    const int rows = min(C::KS, k1 - key0);
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * sizeof(T);
    uint8_t* dst = ring + s * C::kStageBytes;
    if (a.pages.table == nullptr) {
      const int64_t row0 = (static_cast<int64_t>(b) * a.Hkv + g) * a.cap + key0;
      mbar_arrive_expect_tx(&full[s], 2 * bytes);
      bulk_load(dst, a.cache_k + row0 * D, bytes, &full[s]);
      bulk_load(dst + C::kStageBytes / 2, a.cache_v + row0 * D, bytes, &full[s]);
      return;
    }
    issue_paged_rows<T, D>(a.pages, a.cache_k, a.cache_v, a.Hkv, a.cap, a.dev_err, b, g, key0,
                           rows, dst, dst + C::kStageBytes / 2, &full[s]);
  };
  if (tid == 0)
    for (int i = 0; i < kDecStages && i < n_st; ++i) issue(i);

  // per-lane pairs: pair p = lane + 32 kk -> head p / NCH, chunk p % NCH
  const float scale = 1.4426950408889634f * rsqrtf(static_cast<float>(D));
  float qr[kPPMax][C::CH], o[kPPMax][C::CH], m[kPPMax], l[kPPMax];
  const int chunk = lane % C::NCH;
#pragma unroll
  for (int kk = 0; kk < kPPMax; ++kk) {
    const int p = lane + 32 * kk;
    const int h = p / C::NCH;
    m[kk] = -INFINITY;
    l[kk] = 0.f;
#pragma unroll
    for (int e = 0; e < C::CH; ++e) {
      o[kk][e] = 0.f;
      qr[kk][e] = (p < P) ? a.q_ws[(static_cast<int64_t>(b) * a.Hq + g * G + hc0 + h) * D +
                                   chunk * C::CH + e] *
                                scale
                          : 0.f;
    }
  }
  const int PP = (P + 31) / 32;

  for (int it = 0; it < n_st; ++it) {
    const int s = it % kDecStages;
    if (!mbar_wait(&full[s], (it / kDecStages) & 1, &abort_flag, a.dev_err)) break;
    const T* Ks = reinterpret_cast<const T*>(ring + s * C::kStageBytes);
    const T* Vs = reinterpret_cast<const T*>(ring + s * C::kStageBytes + C::kStageBytes / 2);
    const int key_base = k0 + it * C::KS;
    const int rows = min(C::KS, k1 - key_base);
    const int c_lo = warp * C::KW;
    float sc[kPPMax][C::KW];
#pragma unroll
    for (int c = 0; c < C::KW; ++c) {
      const int kr = c_lo + c;
      const bool kv = kr < rows;
      uint4 kraw = kv ? *reinterpret_cast<const uint4*>(Ks + kr * D + chunk * C::CH)
                      : make_uint4(0, 0, 0, 0);
      const T* ke = reinterpret_cast<const T*>(&kraw);
#pragma unroll
      for (int kk = 0; kk < kPPMax; ++kk) {
        if (kk >= PP) break;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < C::CH; ++e) part = fmaf(qr[kk][e], to_f32(ke[e]), part);
#pragma unroll
        for (int off = 1; off < C::NCH; off <<= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        sc[kk][c] = kv ? part : -INFINITY;
      }
    }
#pragma unroll
    for (int kk = 0; kk < kPPMax; ++kk) {
      if (kk >= PP) break;
      float mx = m[kk];
#pragma unroll
      for (int c = 0; c < C::KW; ++c) mx = fmaxf(mx, sc[kk][c]);
      if (mx == -INFINITY) continue;
      const float corr = ex2f(m[kk] - mx);
      l[kk] *= corr;
#pragma unroll
      for (int e = 0; e < C::CH; ++e) o[kk][e] *= corr;
      m[kk] = mx;
#pragma unroll
      for (int c = 0; c < C::KW; ++c) {
        const int kr = c_lo + c;
        if (kr >= rows) break;
        const float pr = ex2f(sc[kk][c] - mx);
        l[kk] += pr;
        const uint4 vraw = *reinterpret_cast<const uint4*>(Vs + kr * D + chunk * C::CH);
        const T* ve = reinterpret_cast<const T*>(&vraw);
#pragma unroll
        for (int e = 0; e < C::CH; ++e) o[kk][e] = fmaf(pr, to_f32(ve[e]), o[kk][e]);
      }
    }
    __syncthreads();  // every warp is done with stage s
    if (tid == 0 && it + kDecStages < n_st) issue(it + kDecStages);
  }

  // merge the four warps: wbuf[warp][p] = (m, l), then o
  float* wm = wbuf;                       // [4][P]
  float* wl = wm + 4 * P;                 // [4][P]
  float* wo = wl + 4 * P;                 // [4][P][CH]
#pragma unroll
  for (int kk = 0; kk < kPPMax; ++kk) {
    const int p = lane + 32 * kk;
    if (kk >= PP || p >= P) break;
    wm[warp * P + p] = m[kk];
    wl[warp * P + p] = l[kk];
#pragma unroll
    for (int e = 0; e < C::CH; ++e) wo[(warp * P + p) * C::CH + e] = o[kk][e];
  }
  __syncthreads();
  const int64_t pbase = ((static_cast<int64_t>(b) * a.Hkv + g) * a.splits + sp) * G + hc0;
  for (int p = tid; p < P; p += kDecThreads) {
    float M = -INFINITY;
    for (int w = 0; w < 4; ++w) M = fmaxf(M, wm[w * P + p]);
    float lsum = 0.f, oacc[C::CH];
#pragma unroll
    for (int e = 0; e < C::CH; ++e) oacc[e] = 0.f;
    for (int w = 0; w < 4; ++w) {
      const float f = (M == -INFINITY) ? 0.f : ex2f(wm[w * P + p] - M);
      lsum += wl[w * P + p] * f;
#pragma unroll
      for (int e = 0; e < C::CH; ++e) oacc[e] += wo[(w * P + p) * C::CH + e] * f;
    }
    const int h = p / C::NCH, ck = p % C::NCH;
    if (ck == 0) {
      a.part_ml[(pbase + h) * 2] = M;
      a.part_ml[(pbase + h) * 2 + 1] = lsum;
    }
#pragma unroll
    for (int e = 0; e < C::CH; ++e) a.part_o[(pbase + h) * D + ck * C::CH + e] = oacc[e];
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(a.tickets + b * a.Hkv + g, 1);
    last_flag = (prev == a.splits * n_hc - 1);
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  // the last CTA of (b, g) merges every split of its G heads in one pass
  const int64_t gbase = (static_cast<int64_t>(b) * a.Hkv + g) * a.splits * G;
  for (int idx = tid; idx < G * D; idx += kDecThreads) {
    const int h = idx / D, i = idx - h * D;
    float M = -INFINITY, lsum = 0.f, acc = 0.f;
#pragma unroll 4
    for (int s2 = 0; s2 < a.splits; ++s2) {
      const int64_t pi = gbase + static_cast<int64_t>(s2) * G + h;
      const float ms = __ldcg(a.part_ml + pi * 2);
      const float ls = __ldcg(a.part_ml + pi * 2 + 1);
      const float os = __ldcg(a.part_o + pi * D + i);
      if (ms == -INFINITY) continue;
      if (ms > M) {
        const float corr = ex2f(M - ms);   // 0 when M is still -inf
        lsum *= corr;
        acc *= corr;
        M = ms;
      }
      const float f = ex2f(ms - M);
      lsum = fmaf(ls, f, lsum);
      acc = fmaf(os, f, acc);
    }
    const float val = (valid_b && lsum > 0.f) ? acc / lsum : 0.f;
    a.out[static_cast<int64_t>(b) * a.Hq * D + (g * G + h) * D + i] = from_f32<T>(val);
  }
  __syncthreads();
  if (tid == 0) {
    a.tickets[b * a.Hkv + g] = 0;
    __threadfence();
    const int prev = atomicAdd(a.tickets + a.B * a.Hkv + b, 1);
    if (prev == a.Hkv - 1) {
      a.tickets[a.B * a.Hkv + b] = 0;
      if (valid_b) a.len[b] = L + 1;
    }
  }
}

template <typename T, int D>
size_t dec_attn_smem(int G) {
  using C = DecCfg<T, D>;
  const int n_hc = dec_head_chunks<T, D>(G);
  const int P = (G + n_hc - 1) / n_hc * C::NCH;
  return 128 + kDecStages * C::kStageBytes + kDecStages * 8 +
         static_cast<size_t>(4 * P * (2 + C::CH)) * 4 + 16;
}

template <typename T, int D>
cudaError_t launch_dec_attn(const DecodeArgs<T>& a, cudaStream_t stream) {
  const size_t smem = dec_attn_smem<T, D>(a.G);
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(decode_attn_kernel<T, D>),
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.Hkv * dec_head_chunks<T, D>(a.G), a.B);
  decode_attn_kernel<T, D><<<grid, kDecThreads, smem, stream>>>(a);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace

namespace {
template <typename T>
cudaError_t launch_rows_copy(T* ck, T* cv, const PageMap& pm, const int32_t* len, const T* kn,
                             const T* vn, int64_t sb, int64_t si, int64_t sg, int B, int Hkv,
                             int d, int64_t cap, int n, int32_t* dev_err, cudaStream_t stream) {
  const int64_t chunks = static_cast<int64_t>(n) * Hkv * (d * sizeof(T) / 16);
  int64_t blocks = (chunks + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  if (blocks < 1) blocks = 1;
  dim3 grid(static_cast<unsigned>(blocks), B);
  kv_append_kernel<T><<<grid, 256, 0, stream>>>(ck, cv, pm, len, kn, vn, sb, si, sg, Hkv, d, cap,
                                                n, dev_err);
  count_launches(1);
  return cudaGetLastError();
}
}  // namespace

template <typename T>
cudaError_t launch_kv_append(T* cache_k, T* cache_v, const PageMap& pm, int32_t* len,
                             const T* k_new, const T* v_new, int B, int Hkv, int d, int64_t cap,
                             int n_new, int32_t* dev_err, cudaStream_t stream) {
  const cudaError_t e = launch_rows_copy<T>(cache_k, cache_v, pm, len, k_new, v_new,
                                            static_cast<int64_t>(n_new) * Hkv, Hkv, 1, B, Hkv, d,
                                            cap, n_new, dev_err, stream);
  if (e != cudaSuccess) return e;
  len_add_kernel<<<(B + 127) / 128, 128, 0, stream>>>(len, B, cap, n_new);
  count_launches(1);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_kv_scatter(T* cache_k, T* cache_v, const PageMap& pm, const T* k_src,
                              const T* v_src, int B, int Hkv, int d, int64_t cap, int S,
                              int32_t* dev_err, cudaStream_t stream) {
  return launch_rows_copy<T>(cache_k, cache_v, pm, nullptr, k_src, v_src,
                             static_cast<int64_t>(Hkv) * S, 1, S, B, Hkv, d, cap, S, dev_err,
                             stream);
}

bool decode_pre_fits(int G, int d, int K, int es) {
  const size_t bytes = es == 2 ? pre_smem<bf16>(G, d, K).bytes_no_w
                               : pre_smem<float>(G, d, K).bytes_no_w;
  return bytes <= 227 * 1024;
}

template <typename T>
cudaError_t launch_decode_step(const DecodeArgs<T>& a, cudaStream_t stream) {
  cudaError_t e;
  auto mark = [&](int i) {
    if (a.phase_events) cudaEventRecord(static_cast<cudaEvent_t>(a.phase_events[i]), stream);
  };
  mark(0);
  if (a.W) {
    if (decode_use_gemv(a.B, a.E, sizeof(T)) && a.e_splits == 1) {
      if ((e = launch_gemv<T>(a.x_t, a.W, a.proj_part, a.B, a.E, a.N, stream)) != cudaSuccess)
        return e;
    } else if (decode_use_proj_tc(a.E, sizeof(T)) && a.e_splits == a.E / kDpK) {
      if constexpr (sizeof(T) == 2) {
        if ((e = launch_decode_proj_tc(a.x_t, a.W, a.proj_part, a.B, a.E, a.N, a.dev_err,
                                       stream)) != cudaSuccess)
          return e;
      }
    } else {
      const int e_len = decode_proj_e_len(a.E, a.e_splits);
      dim3 grid((a.N + kPN - 1) / kPN, a.e_splits, (a.B + kPB - 1) / kPB);
      decode_proj_kernel<T><<<grid, 256, 0, stream>>>(a.x_t, a.W, a.proj_part, a.B, a.E, a.N, e_len);
    }
    count_launches(1);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  mark(1);
  {
    const PreSmem Ls = pre_smem<T>(a.G, a.d, a.K);
    const int stage_wt = Ls.bytes <= kPreSmemMax;
    const size_t smem = stage_wt ? Ls.bytes : Ls.bytes_no_w;
    if (smem > 48 * 1024) {
      e = allow_smem(reinterpret_cast<const void*>(decode_pre_kernel<T>),
                               static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    e = launch_pdl(decode_pre_kernel<T>, dim3(a.Hkv, a.B), dim3(kPreThreads), smem, stream, a,
                   stage_wt);
    count_launches(1);
    if (e != cudaSuccess || (e = cudaGetLastError()) != cudaSuccess) return e;
  }
  mark(2);
  if constexpr (sizeof(T) == 2) {
    if (a.G <= 16 && a.d >= 32) {
      e = launch_decode_attn_tc(a, stream);
      mark(3);
      return e;
    }
  }
  switch (a.d) {
    case 16: e = launch_dec_attn<T, 16>(a, stream); break;
    case 32: e = launch_dec_attn<T, 32>(a, stream); break;
    case 64: e = launch_dec_attn<T, 64>(a, stream); break;
    case 128: e = launch_dec_attn<T, 128>(a, stream); break;
    default: e = cudaErrorInvalidValue;
  }
  mark(3);
  return e;
}

template cudaError_t launch_kv_append<float>(float*, float*, const PageMap&, int32_t*,
                                             const float*, const float*, int, int, int, int64_t,
                                             int, int32_t*, cudaStream_t);
template cudaError_t launch_kv_append<bf16>(bf16*, bf16*, const PageMap&, int32_t*, const bf16*,
                                            const bf16*, int, int, int, int64_t, int, int32_t*,
                                            cudaStream_t);
template cudaError_t launch_kv_scatter<float>(float*, float*, const PageMap&, const float*,
                                              const float*, int, int, int, int64_t, int, int32_t*,
                                              cudaStream_t);
template cudaError_t launch_kv_scatter<bf16>(bf16*, bf16*, const PageMap&, const bf16*,
                                             const bf16*, int, int, int, int64_t, int, int32_t*,
                                             cudaStream_t);
template cudaError_t launch_decode_step<float>(const DecodeArgs<float>&, cudaStream_t);
template cudaError_t launch_decode_step<bf16>(const DecodeArgs<bf16>&, cudaStream_t);

}  // namespace ccgqa
