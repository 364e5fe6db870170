// Attention backward on the 5th-generation tensor core (bf16): the gradient of
// the causal grouped-query attention of "Compressed Convolutional Attention"
// (section CCGQA; Resultaten 2: the layer is trained, so its backward pass
// runs on the same hardware), for power-of-two groups of at most 64 heads.
//
// Inputs: q [B, S, Hq, d], k, v [B, Hkv, S, d], the forward output o and the
// upstream gradient dO [B, S, Hq, d] (bf16), and the forward's log-sum-exp in
// base 2 per query row, lse2 = log2(sum_s 2^(c s_ts)) with c = log2(e) / sqrt(d),
// stored negated in the packed row order of the forward (row t G + head in
// group, a stride of ld floats per (sequence, kv group)); D is stored negated
// the same way, so that each score costs one packed FMA before the exponential
// and one packed add and multiply after it.  With P = 2^(c S - lse2) the
// softmax of the scores S = q k^T and D = rowsum(dO o):
//   dP = dO v^T,  dS = P (dP - D),  dq = dS k / sqrt(d),
//   dk = dS^T q / sqrt(d),  dv = P^T dO   (summed over the G heads of a group).
//
// Two kernels, both built like the forward kernel (TMA producer warp, one MMA
// issuer thread per 128-row tile, four softmax warps per tile with one row per
// thread and TMEM lane, no cluster multicast, every wait bounded):
//   dq pass   query-major: per 128-row packed query tile (T tiles per CTA),
//             K/V tiles of 128 keys as two 64-key halves.  S = Q K^T and
//             dP = dO V^T (SS) into TMEM; the softmax warps form P from lse2
//             (no running max: the forward fixed it), then dS, written as bf16
//             over the dP buffer; dQ += dS K (TS, K read MN-major).  They also
//             form D for their rows (read by the second kernel).
//   dkv pass  key-major: per 128-key tile (T tiles per CTA), the packed query
//             rows that see it in halves of 64 rows (Q and dO halves, lse2 and
//             D of the half by bulk copy), each worked as two 32-row
//             sub-halves in two TMEM buffers per tile.  S^T = K Q^T,
//             dP^T = V dO^T; P^T is written as bf16 over S^T and dS^T over
//             dP^T; dV += P^T dO and dK += dS^T Q (TS) while the next
//             sub-half's scores go into the other buffer.  A half holds rows of
//             all G heads, so the group's sum comes from the MMA itself.  A key
//             tile's halves are cut into chunks, one CTA each, whose dK / dV
//             are added atomically into zeroed buffers.
// The 1 / sqrt(d) of dq and dk is applied at the store; P and dS are rounded
// to bf16 for the MMAs, everything else is fp32.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr float kLog2eB = 1.4426950408889634f;

template <int D>
struct BwdTcCfg {
  static constexpr int kPanelCols = (D == 32) ? 32 : 64;      // elements per swizzle row
  static constexpr int kPanels = D / kPanelCols;
  static constexpr uint32_t kRowBytes = kPanelCols * 2;
  static constexpr uint32_t kSwz = (D == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;
  static constexpr uint32_t kPanel128 = 128 * kRowBytes;      // one panel of a 128-row tile
  static constexpr uint32_t kPanel64 = 64 * kRowBytes;        // one panel of a 64-row half
  static constexpr uint32_t kTile = 128 * D * 2;
  static constexpr uint32_t kHalf = 64 * D * 2;
  static constexpr int kTiles = (D == 128) ? 1 : 2;
  static constexpr int kThreads = 128 + 128 * kTiles;
  static constexpr uint32_t kTmemCols = 512;
  // dq pass shared memory: Q and dO tiles, then the K and V ring
  static constexpr int kQStages = (D == 128) ? 2 : (D == 64 ? 3 : 4);
  static constexpr uint32_t kQOffQ = 0;
  static constexpr uint32_t kQOffDO = kQOffQ + kTiles * kTile;
  static constexpr uint32_t kQOffK = kQOffDO + kTiles * kTile;
  static constexpr uint32_t kQOffV = kQOffK + kQStages * kTile;
  static constexpr uint32_t kQOffBar = kQOffV + kQStages * kTile;
  static constexpr size_t kQSmem = kQOffBar + 256 + 1024;
  // dkv pass shared memory: K and V tiles, then the ring of Q / dO halves and
  // their lse2 / D rows
  static constexpr int kKStages = (D == 128) ? 3 : 4;
  static constexpr uint32_t kKOffK = 0;
  static constexpr uint32_t kKOffV = kKOffK + kTiles * kTile;
  static constexpr uint32_t kKOffQ = kKOffV + kTiles * kTile;
  static constexpr uint32_t kKOffDO = kKOffQ + kKStages * kHalf;
  static constexpr uint32_t kKOffL = kKOffDO + kKStages * kHalf;   // [stage][-lse2 64 | -D 64]
  static constexpr uint32_t kKOffBar = kKOffL + kKStages * 512;
  static constexpr size_t kKSmem = kKOffBar + 256 + 1024;
  // TMEM columns.  dq pass: S and dP (64 each) per tile, then dQ per tile.
  // dkv pass: per tile two buffers of S^T | dP^T (32 + 32 columns), then
  // dV | dK per tile.
  __device__ static constexpr uint32_t col_s(int x) { return x * 128; }
  __device__ static constexpr uint32_t col_dp(int x) { return x * 128 + 64; }
  __device__ static constexpr uint32_t col_dq(int x) { return kTiles * 128 + x * D; }
  __device__ static constexpr uint32_t col_dkv_buf(int x, int b) { return x * 128 + b * 64; }
  __device__ static constexpr uint32_t col_dkv_v(int x) { return kTiles * 128 + x * 2 * D; }
  __device__ static constexpr uint32_t col_dkv_k(int x) { return kTiles * 128 + x * 2 * D + D; }
  static_assert(kTiles * 128 + kTiles * 2 * D <= 512, "TMEM columns");
  static_assert(kQSmem <= 227 * 1024 && kKSmem <= 227 * 1024, "shared memory");
};

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Four consecutive floats of shared memory, read where they are used (volatile:
// not hoisted, so a row's 64 column constants never sit in registers at once).
__device__ __forceinline__ float4 lds4(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(smem_addr(p)));
  return v;
}

// Packed fp32 pairs on the FMA pipe (one instruction for two values).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)),
        "l"(*reinterpret_cast<const uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<const uint64_t*>(&a)), "l"(*reinterpret_cast<const uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h2);
}

// S (or dP) of a tile: A is the 128-row tile at a_base (K-major, panels of 128
// rows), B the 64-row operand at b_base with panels b_panel bytes apart;
// K = d in steps of 16.
template <int D>
__device__ __forceinline__ void mma_rows_x_cols(uint32_t d_tmem, uint32_t a_base, uint32_t b_base,
                                                uint32_t b_panel, uint32_t idesc) {
  using C = BwdTcCfg<D>;
#pragma unroll
  for (int k = 0; k < D / 16; ++k) {
    const int p = (k * 16) / C::kPanelCols;
    const uint32_t in = ((k * 16) % C::kPanelCols) * 2;
    const uint64_t ad = make_smem_desc(a_base + p * C::kPanel128 + in, 16, C::kSbo, C::kSwz);
    const uint64_t bd = make_smem_desc(b_base + p * b_panel + in, 16, C::kSbo, C::kSwz);
    mma_ss(d_tmem, ad, bd, idesc, k > 0 ? 1u : 0u);
  }
}

// acc (+)= A_tmem B: A is 128 rows x 64 bf16 in TMEM (32 columns of pairs),
// B the 64-row operand at b_base read MN-major (d contiguous, panels b_panel
// bytes apart); K = 64 in steps of 16.
template <int D>
__device__ __forceinline__ void mma_tmem_x_rows(uint32_t acc, uint32_t a_tmem, uint32_t b_base,
                                                uint32_t b_panel, uint32_t idesc, bool first) {
  using C = BwdTcCfg<D>;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const uint64_t bd = make_smem_desc(b_base + kk * 16 * C::kRowBytes, b_panel, C::kSbo, C::kSwz);
    mma_ts(acc, a_tmem + kk * 8, bd, idesc, (!first || kk > 0) ? 1u : 0u);
  }
}

// ================================================================ dq pass
template <int D>
__global__ void __launch_bounds__(BwdTcCfg<D>::kThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                          const __grid_constant__ CUtensorMap tmDO,
                          const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const bf16* __restrict__ o,
                          const bf16* __restrict__ dout, const float* __restrict__ lse,
                          float* __restrict__ dsum, float* __restrict__ dq, int B, int S, int Hq,
                          int Hkv, int G_log2, int n_groups, int causal, int64_t ld,
                          int32_t* dev_err) {
  pdl_enter();
  using C = BwdTcCfg<D>;
  constexpr int T = C::kTiles;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kQOffBar);
  uint64_t* q_full = bars;                        // Q and dO tiles
  uint64_t* kv_full = q_full + 1;                 // [kQStages]
  uint64_t* kv_empty = kv_full + C::kQStages;     // [kQStages], one commit per tile
  uint64_t* s_full = kv_empty + C::kQStages;      // [T]
  uint64_t* dp_full = s_full + T;                 // [T]
  uint64_t* ds_full = dp_full + T;                // [T], 128 arrivals
  uint64_t* dq_done = ds_full + T;                // [T]
  uint64_t* drain = dq_done + T;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = 1 << G_log2;
  const int BH = B * Hkv;
  const int grp = n_groups - 1 - static_cast<int>(blockIdx.x) / BH;   // longest first
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int b = bg / Hkv, g = bg % Hkv;
  const int pos_per_tile = 128 >> G_log2;
  const int t0 = grp * T * pos_per_tile;
  const int t_last = min(t0 + T * pos_per_tile - 1, S - 1);
  const int n_kv = causal ? (t_last / 128 + 1) : (S + 127) / 128;
  const int n_h = 2 * n_kv;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kQStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], T);
    }
    for (int x = 0; x < T; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&dp_full[x], 1);
      mbar_init(&ds_full[x], 128);
      mbar_init(&dq_done[x], 1);
    }
    mbar_init(drain, T);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmDO);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, 2 * T * C::kTile);
#pragma unroll
      for (int x = 0; x < T; ++x)
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_5d(smem + C::kQOffQ + x * C::kTile + p * C::kPanel128, &tmQ, q_full,
                      p * C::kPanelCols, 0, g, t0 + x * pos_per_tile, b);
          tma_load_5d(smem + C::kQOffDO + x * C::kTile + p * C::kPanel128, &tmDO, q_full,
                      p * C::kPanelCols, 0, g, t0 + x * pos_per_tile, b);
        }
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::kQStages;
        if (!mbar_wait(&kv_empty[st], ((j / C::kQStages) & 1) ^ 1, &abort_flag, dev_err)) break;
        mbar_arrive_expect_tx(&kv_full[st], 2 * C::kTile);
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_3d(smem + C::kQOffK + st * C::kTile + p * C::kPanel128, &tmK, &kv_full[st],
                      p * C::kPanelCols, j * 128, bg);
          tma_load_3d(smem + C::kQOffV + st * C::kTile + p * C::kPanel128, &tmV, &kv_full[st],
                      p * C::kPanelCols, j * 128, bg);
        }
      }
    }
  } else if (warp >= 1 && warp <= T) {
    // ------------------------------------------------------------ MMA issuer
    // Half k = 2 j + h: S(k) and dP(k); after the softmax wrote dS(k): dQ(k),
    // then S(k+1) into the S buffer it has read, and, once dQ(k) has read
    // dS(k), dP(k+1) into the dP buffer.
    if (lane == 0) {
      const int x = warp - 1;
      const uint32_t idesc_s = make_idesc_bf16(128, 64, false);
      const uint32_t idesc_o = make_idesc_bf16(128, D, true);
      const uint32_t q_base = smem_addr(smem + C::kQOffQ) + x * C::kTile;
      const uint32_t do_base = smem_addr(smem + C::kQOffDO) + x * C::kTile;
      auto kv_half = [&](uint32_t off, int k) {
        return smem_addr(smem + off + ((k >> 1) % C::kQStages) * C::kTile) +
               (k & 1) * 64 * C::kRowBytes;
      };
      auto issue_s = [&](int k) {
        mma_rows_x_cols<D>(tmem + C::col_s(x), q_base, kv_half(C::kQOffK, k), C::kPanel128, idesc_s);
        mma_commit(&s_full[x]);
      };
      auto issue_dp = [&](int k) {
        mma_rows_x_cols<D>(tmem + C::col_dp(x), do_base, kv_half(C::kQOffV, k), C::kPanel128,
                           idesc_s);
        mma_commit(&dp_full[x]);
      };
      bool ok = mbar_wait(q_full, 0, &abort_flag, dev_err) &&
                mbar_wait(&kv_full[0], 0, &abort_flag, dev_err);
      if (ok) {
        tc_fence_after();
        issue_s(0);
        issue_dp(0);
      }
      for (int k = 0; ok && k < n_h; ++k) {
        if (!mbar_wait(&ds_full[x], k & 1, &abort_flag, dev_err)) break;
        tc_fence_after();
        mma_tmem_x_rows<D>(tmem + C::col_dq(x), tmem + C::col_dp(x), kv_half(C::kQOffK, k),
                           C::kPanel128, idesc_o, k == 0);
        mma_commit(&dq_done[x]);
        if (k & 1) mma_commit(&kv_empty[(k >> 1) % C::kQStages]);
        if (k + 1 < n_h) {
          const int jn = (k + 1) >> 1;
          if (((k + 1) & 1) == 0 &&
              !mbar_wait(&kv_full[jn % C::kQStages], (jn / C::kQStages) & 1, &abort_flag, dev_err))
            break;
          tc_fence_after();
          issue_s(k + 1);
          if (!mbar_wait(&dq_done[x], k & 1, &abort_flag, dev_err)) break;
          tc_fence_after();
          issue_dp(k + 1);
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // tile row == TMEM lane
    const int t = t0 + x * pos_per_tile + (r >> G_log2);
    const int hl = r & (G - 1);
    const bool row_in = t < S;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int64_t prow = static_cast<int64_t>(bg) * ld + (static_cast<int64_t>(t) << G_log2) + hl;
    const int64_t grow = ((static_cast<int64_t>(b) * S + t) * Hq + g * G + hl) * D;
    // D = rowsum(dO o) of this row (bf16 inputs, fp32 sum), kept for the dkv pass
    float nlse = 0.f, Dr = 0.f;   // -lse2, D
    if (row_in) {
      nlse = lse[prow];
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        const uint4 a4 = *reinterpret_cast<const uint4*>(dout + grow + i * 8);
        const uint4 o4 = *reinterpret_cast<const uint4*>(o + grow + i * 8);
        const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a4);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&o4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 af = __bfloat1622float2(a2[e]), of = __bfloat1622float2(o2[e]);
          acc[e] = fmaf(af.x, of.x, acc[e]);
          acc[e] = fmaf(af.y, of.y, acc[e]);
        }
      }
      Dr = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      dsum[prow] = -Dr;
    }
    const float2 nl2 = make_float2(nlse, nlse), nd2 = make_float2(-Dr, -Dr);
    const float c = kLog2eB * rsqrtf(static_cast<float>(D));
    const float2 c2 = make_float2(c, c);
    bool ok = true;
    for (int k = 0; k < n_h; ++k) {
      const int kb = k * 64;
      int lim = S - 1 - kb;                        // keys kb + e are visible when e <= lim
      if (causal) lim = min(lim, t - kb);
      if (!row_in) lim = -1;
      const bool full = __all_sync(0xffffffffu, lim >= 63);
      if (!mbar_wait(&s_full[x], k & 1, &abort_flag, dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float p[64];
      tmem_ld32(trow + C::col_s(x), *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(trow + C::col_s(x) + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 64; e += 2) {
        const float2 a2 = ffma2(make_float2(p[e], p[e + 1]), c2, nl2);
        p[e] = ex2f(a2.x);
        p[e + 1] = ex2f(a2.y);
      }
      if (!full) {
#pragma unroll
        for (int e = 0; e < 64; ++e) p[e] = (e <= lim) ? p[e] : 0.f;
      }
      if (!mbar_wait(&dp_full[x], k & 1, &abort_flag, dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dp[32], ds[16];
        tmem_ld32(trow + C::col_dp(x) + ch * 32, dp);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float2 d2 = fmul2(make_float2(p[ch * 32 + 2 * e], p[ch * 32 + 2 * e + 1]),
                                  fadd2(make_float2(__uint_as_float(dp[2 * e]),
                                                    __uint_as_float(dp[2 * e + 1])),
                                        nd2));
          ds[e] = pack2(d2.x, d2.y);
        }
        tmem_st16(trow + C::col_dp(x) + ch * 16, ds);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ds_full[x]);
    }
    if (ok && mbar_wait(&dq_done[x], (n_h - 1) & 1, &abort_flag, dev_err)) {
      tc_fence_after();
      const float sc = rsqrtf(static_cast<float>(D));
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(trow + C::col_dq(x) + cc * 32, v);
        tmem_wait_ld();
        if (row_in) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dq + grow + cc * 32 + e) =
                make_float4(__uint_as_float(v[e]) * sc, __uint_as_float(v[e + 1]) * sc,
                            __uint_as_float(v[e + 2]) * sc, __uint_as_float(v[e + 3]) * sc);
        }
      }
    }
  }

  if (abort_flag && warp >= 1 && warp <= T && lane == 0) {
    mma_commit(drain);
    const long long t0c = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - t0c < kWaitLimitCycles) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ================================================================ dkv pass
// Each 64-row query half is worked as two 32-row sub-halves, and each tile has
// two TMEM buffers (S^T | dP^T, 32 columns each, P^T and dS^T written back as
// bf16 over them), so the next sub-half's scores are computed into the other
// buffer while the dV / dK MMAs of this one run.
template <int D>
__global__ void __launch_bounds__(BwdTcCfg<D>::kThreads, 1)
    attn_bwd_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQh,
                           const __grid_constant__ CUtensorMap tmDOh,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV,
                           const float* __restrict__ lse, const float* __restrict__ dsum,
                           float* __restrict__ dk, float* __restrict__ dv, int B, int S, int Hkv,
                           int G_log2, int causal, int64_t ld, int chunk_halves, int max_chunks,
                           int32_t* dev_err) {
  pdl_enter();
  using C = BwdTcCfg<D>;
  constexpr int T = C::kTiles;
  // CTA = (key group, chunk of at most chunk_halves query halves, sequence x
  // kv group); the chunks' dK / dV are summed atomically into zeroed buffers
  const int BH = B * Hkv;
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int chunk = (static_cast<int>(blockIdx.x) / BH) % max_chunks;
  const int kgrp = static_cast<int>(blockIdx.x) / BH / max_chunks;   // ascending: longest first
  const int k_start = kgrp * T * 128;
  const int64_t rows_all = static_cast<int64_t>(S) << G_log2;   // packed query rows of (b, g)
  const int u_first = causal ? static_cast<int>((static_cast<int64_t>(k_start) << G_log2) >> 6) : 0;
  const int n_h_all = static_cast<int>((rows_all + 63) >> 6) - u_first;
  if (chunk * chunk_halves >= n_h_all) return;   // nothing left for this chunk
  const int u0 = u_first + chunk * chunk_halves;
  const int n_h = min(chunk_halves, n_h_all - chunk * chunk_halves);   // 64-row halves
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kKOffBar);
  uint64_t* kv_full = bars;                       // K and V tiles
  uint64_t* h_full = kv_full + 1;                 // [kKStages] Q / dO halves, lse2 / D
  uint64_t* h_empty = h_full + C::kKStages;       // [kKStages], one commit per tile
  uint64_t* st_full = h_empty + C::kKStages;      // [T][2] S^T and dP^T of a buffer
  uint64_t* ds_full = st_full + 2 * T;            // [T][2] 128 arrivals: P^T, dS^T written
  uint64_t* o_done = ds_full + 2 * T;             // [T][2] dV / dK of a buffer complete
  uint64_t* drain = o_done + 2 * T;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bg / Hkv, g = bg % Hkv;
  const int n_s = 2 * n_h;                                      // 32-row sub-halves
  const int pos_per_half = 64 >> G_log2;

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < C::kKStages; ++s) {
      mbar_init(&h_full[s], 1);
      mbar_init(&h_empty[s], T);
    }
    for (int i = 0; i < 2 * T; ++i) {
      mbar_init(&st_full[i], 1);
      mbar_init(&ds_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, T);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmQh);
      prefetch_tensormap(&tmDOh);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(kv_full, 2 * T * C::kTile);
#pragma unroll
      for (int x = 0; x < T; ++x)
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_3d(smem + C::kKOffK + x * C::kTile + p * C::kPanel128, &tmK, kv_full,
                      p * C::kPanelCols, k_start + x * 128, bg);
          tma_load_3d(smem + C::kKOffV + x * C::kTile + p * C::kPanel128, &tmV, kv_full,
                      p * C::kPanelCols, k_start + x * 128, bg);
        }
      const float* lrow = lse + static_cast<int64_t>(bg) * ld;
      const float* drow = dsum + static_cast<int64_t>(bg) * ld;
      for (int i = 0; i < n_h; ++i) {
        const int st = i % C::kKStages, u = u0 + i;
        if (!mbar_wait(&h_empty[st], ((i / C::kKStages) & 1) ^ 1, &abort_flag, dev_err)) break;
        mbar_arrive_expect_tx(&h_full[st], 2 * C::kHalf + 512);
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_5d(smem + C::kKOffQ + st * C::kHalf + p * C::kPanel64, &tmQh, &h_full[st],
                      p * C::kPanelCols, 0, g, u * pos_per_half, b);
          tma_load_5d(smem + C::kKOffDO + st * C::kHalf + p * C::kPanel64, &tmDOh, &h_full[st],
                      p * C::kPanelCols, 0, g, u * pos_per_half, b);
        }
        bulk_load(smem + C::kKOffL + st * 512, lrow + u * 64, 256, &h_full[st]);
        bulk_load(smem + C::kKOffL + st * 512 + 256, drow + u * 64, 256, &h_full[st]);
      }
    }
  } else if (warp >= 1 && warp <= T) {
    // ------------------------------------------------------------ MMA issuer
    // Sub-half s (buffer s & 1): S^T(s) = K Q_s^T and dP^T(s) = V dO_s^T
    // (M = 128 keys, N = 32 rows); once the softmax wrote P^T(s) / dS^T(s):
    // dV += P^T(s) dO_s and dK += dS^T(s) Q_s (TS, K = 32), and, once those
    // have read the buffer, S^T(s + 2) / dP^T(s + 2) into it.
    if (lane == 0) {
      const int x = warp - 1;
      const uint32_t idesc_s = make_idesc_bf16(128, 32, false);
      const uint32_t idesc_o = make_idesc_bf16(128, D, true);
      const uint32_t k_base = smem_addr(smem + C::kKOffK) + x * C::kTile;
      const uint32_t v_base = smem_addr(smem + C::kKOffV) + x * C::kTile;
      // rows of sub-half s inside its half's stage
      auto sub_at = [&](uint32_t off, int s) {
        return smem_addr(smem + off + ((s >> 1) % C::kKStages) * C::kHalf) +
               (s & 1) * 32 * C::kRowBytes;
      };
      auto issue_st = [&](int s) {
        const uint32_t buf = C::col_dkv_buf(x, s & 1);
        mma_rows_x_cols<D>(tmem + buf, k_base, sub_at(C::kKOffQ, s), C::kPanel64, idesc_s);
        mma_rows_x_cols<D>(tmem + buf + 32, v_base, sub_at(C::kKOffDO, s), C::kPanel64, idesc_s);
        mma_commit(&st_full[x * 2 + (s & 1)]);
      };
      auto issue_out = [&](int s) {
        const uint32_t buf = C::col_dkv_buf(x, s & 1);
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const uint64_t bdo =
              make_smem_desc(sub_at(C::kKOffDO, s) + kk * 16 * C::kRowBytes, C::kPanel64, C::kSbo, C::kSwz);
          mma_ts(tmem + C::col_dkv_v(x), tmem + buf + kk * 8, bdo, idesc_o, (s > 0 || kk > 0) ? 1u : 0u);
          const uint64_t bq =
              make_smem_desc(sub_at(C::kKOffQ, s) + kk * 16 * C::kRowBytes, C::kPanel64, C::kSbo, C::kSwz);
          mma_ts(tmem + C::col_dkv_k(x), tmem + buf + 32 + kk * 8, bq, idesc_o,
                 (s > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[x * 2 + (s & 1)]);
        if (s & 1) mma_commit(&h_empty[(s >> 1) % C::kKStages]);
      };
      bool ok = mbar_wait(kv_full, 0, &abort_flag, dev_err) &&
                mbar_wait(&h_full[0], 0, &abort_flag, dev_err);
      if (ok) {
        tc_fence_after();
        issue_st(0);
        issue_st(1);
      }
      for (int s = 0; ok && s < n_s; ++s) {
        const int bsel = x * 2 + (s & 1);
        if (!mbar_wait(&ds_full[bsel], (s >> 1) & 1, &abort_flag, dev_err)) break;
        tc_fence_after();
        issue_out(s);
        if (s + 2 < n_s) {
          // S^T(s + 2) reuses this buffer: the dV / dK MMAs just issued read it
          if (((s + 2) & 1) == 0 &&
              !mbar_wait(&h_full[((s + 2) >> 1) % C::kKStages], (((s + 2) >> 1) / C::kKStages) & 1,
                         &abort_flag, dev_err))
            break;
          if (!mbar_wait(&o_done[bsel], (s >> 1) & 1, &abort_flag, dev_err)) break;
          tc_fence_after();
          issue_st(s + 2);
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // key row == TMEM lane
    const int s_pos = k_start + x * 128 + r;
    const bool key_in = s_pos < S;
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float c = kLog2eB * rsqrtf(static_cast<float>(D));
    bool ok = true;
    for (int s = 0; s < n_s; ++s) {
      const int i = s >> 1, st = i % C::kKStages;
      const int64_t row0 = static_cast<int64_t>(u0 + i) * 64 + (s & 1) * 32;   // first row
      // columns e of the sub-half are visible when lo <= e < hi
      int lo = 0;
      if (causal) {
        const int64_t first = (static_cast<int64_t>(s_pos) << G_log2) - row0;
        lo = first <= 0 ? 0 : (first >= 32 ? 32 : static_cast<int>(first));
      }
      const int64_t left = rows_all - row0;
      const int hi = left >= 32 ? 32 : (left <= 0 ? 0 : static_cast<int>(left));
      if (!key_in) lo = 32;
      const bool full = __all_sync(0xffffffffu, lo == 0 && hi == 32);
      const int bsel = x * 2 + (s & 1);
      const uint32_t buf = C::col_dkv_buf(x, s & 1);
      // -lse2 / -D of the half (h_full: the bulk copies have landed)
      if (!mbar_wait(&h_full[st], (i / C::kKStages) & 1, &abort_flag, dev_err) ||
          !mbar_wait(&st_full[bsel], (s >> 1) & 1, &abort_flag, dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float* Ls = reinterpret_cast<const float*>(smem + C::kKOffL + st * 512) + (s & 1) * 32;
      const float* Ds = Ls + 64;
      uint32_t sv[32], dpv[32], pt[16], dt[16];
      tmem_ld32(trow + buf, sv);
      tmem_ld32(trow + buf + 32, dpv);
      tmem_wait_ld();
      // Ls / Ds hold -lse2 and -D per column: p = 2^(c s - lse2), ds = p (dp - D)
      const float2 c2 = make_float2(c, c);
      if (full) {
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const float4 l4 = lds4(Ls + e4);
          const float4 d4 = lds4(Ds + e4);
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int e = e4 + 2 * u;
            const float2 a2 = ffma2(make_float2(__uint_as_float(sv[e]), __uint_as_float(sv[e + 1])),
                                    c2, u ? make_float2(l4.z, l4.w) : make_float2(l4.x, l4.y));
            const float2 p2 = make_float2(ex2f(a2.x), ex2f(a2.y));
            const float2 d2 =
                fmul2(p2, fadd2(make_float2(__uint_as_float(dpv[e]), __uint_as_float(dpv[e + 1])),
                                u ? make_float2(d4.z, d4.w) : make_float2(d4.x, d4.y)));
            pt[e / 2] = pack2(p2.x, p2.y);
            dt[e / 2] = pack2(d2.x, d2.y);
          }
        }
      } else {
        // columns outside [lo, hi) are masked (past the sequence, the padding's
        // -lse2 / -D may hold anything, so the results are selected, not scaled)
#pragma unroll
        for (int e4 = 0; e4 < 32; e4 += 4) {
          const float4 l4 = lds4(Ls + e4);
          const float4 d4 = lds4(Ds + e4);
          const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
          const float dv4[4] = {d4.x, d4.y, d4.z, d4.w};
          float pe[4], de[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = e4 + u;
            const bool vis = e >= lo && e < hi;
            const float pv = ex2f(fmaf(__uint_as_float(sv[e]), c, lv[u]));
            pe[u] = vis ? pv : 0.f;
            de[u] = vis ? pv * (__uint_as_float(dpv[e]) + dv4[u]) : 0.f;
          }
          pt[e4 / 2] = pack2(pe[0], pe[1]);
          pt[e4 / 2 + 1] = pack2(pe[2], pe[3]);
          dt[e4 / 2] = pack2(de[0], de[1]);
          dt[e4 / 2 + 1] = pack2(de[2], de[3]);
        }
      }
      tmem_st16(trow + buf, pt);
      tmem_st16(trow + buf + 32, dt);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&ds_full[bsel]);
    }
    // the last sub-half's dV / dK complete after all earlier ones
    if (ok && n_s > 0 &&
        mbar_wait(&o_done[x * 2 + ((n_s - 1) & 1)], ((n_s - 1) >> 1) & 1, &abort_flag, dev_err)) {
      tc_fence_after();
      const float sc = rsqrtf(static_cast<float>(D));
      const int64_t krow = (static_cast<int64_t>(bg) * S + s_pos) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t vv[32], kv[32];
        tmem_ld32(trow + C::col_dkv_v(x) + cc * 32, vv);
        tmem_ld32(trow + C::col_dkv_k(x) + cc * 32, kv);
        tmem_wait_ld();
        if (key_in) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            atomicAdd(reinterpret_cast<float4*>(dv + krow + cc * 32 + e),
                      make_float4(__uint_as_float(vv[e]), __uint_as_float(vv[e + 1]),
                                  __uint_as_float(vv[e + 2]), __uint_as_float(vv[e + 3])));
            atomicAdd(reinterpret_cast<float4*>(dk + krow + cc * 32 + e),
                      make_float4(__uint_as_float(kv[e]) * sc, __uint_as_float(kv[e + 1]) * sc,
                                  __uint_as_float(kv[e + 2]) * sc, __uint_as_float(kv[e + 3]) * sc));
          }
        }
      }
    }
  }

  if (abort_flag && warp >= 1 && warp <= T && lane == 0) {
    mma_commit(drain);
    const long long t0c = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - t0c < kWaitLimitCycles) {
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// q / dO [B, S, Hq, d] as (d, G, Hkv, S, B): a box (panel, G, 1, rows / G, 1)
// lands as `rows` packed rows (position, head in group).
bool packed_rows_map(CUtensorMap* m, const void* base, const AttnBwdTcArgs& a, int panel_cols,
                     int rows, CUtensorMapSwizzle swz) {
  const uint64_t dims[5] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.G),
                            static_cast<uint64_t>(a.Hkv), static_cast<uint64_t>(a.S),
                            static_cast<uint64_t>(a.B)};
  const uint64_t st[4] = {static_cast<uint64_t>(a.d) * 2, static_cast<uint64_t>(a.G) * a.d * 2,
                          static_cast<uint64_t>(a.Hq) * a.d * 2,
                          static_cast<uint64_t>(a.S) * a.Hq * a.d * 2};
  const uint32_t box[5] = {static_cast<uint32_t>(panel_cols), static_cast<uint32_t>(a.G), 1,
                           static_cast<uint32_t>(rows / a.G), 1};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, base, dims, st, box, swz);
}

// k / v [B, Hkv, S, d] as (d, S, B Hkv) in boxes of 128 keys (keys past S read zero).
bool key_rows_map(CUtensorMap* m, const void* base, const AttnBwdTcArgs& a, int panel_cols,
                  CUtensorMapSwizzle swz) {
  const uint64_t dims[3] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(a.S),
                            static_cast<uint64_t>(a.B) * a.Hkv};
  const uint64_t st[2] = {static_cast<uint64_t>(a.d) * 2, static_cast<uint64_t>(a.S) * a.d * 2};
  const uint32_t box[3] = {static_cast<uint32_t>(panel_cols), 128, 1};
  return encode_tensor_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, st, box, swz);
}

template <int D>
cudaError_t launch_bwd_tc(const AttnBwdTcArgs& a, cudaStream_t stream) {
  using C = BwdTcCfg<D>;
  const CUtensorMapSwizzle swz = (D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  int G_log2 = 0;
  while ((1 << G_log2) < a.G) ++G_log2;
  CUtensorMap tmQ, tmDO, tmQh, tmDOh, tmK, tmV;
  if (!packed_rows_map(&tmQ, a.q, a, C::kPanelCols, 128, swz) ||
      !packed_rows_map(&tmDO, a.dout, a, C::kPanelCols, 128, swz) ||
      !packed_rows_map(&tmQh, a.q, a, C::kPanelCols, 64, swz) ||
      !packed_rows_map(&tmDOh, a.dout, a, C::kPanelCols, 64, swz) ||
      !key_rows_map(&tmK, a.k, a, C::kPanelCols, swz) ||
      !key_rows_map(&tmV, a.v, a, C::kPanelCols, swz))
    return cudaErrorInvalidValue;
  const int BH = a.B * a.Hkv;
  // dq pass
  {
    const int pos_per_cta = C::kTiles * (128 >> G_log2);
    const int n_groups = (a.S + pos_per_cta - 1) / pos_per_cta;
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(attn_bwd_dq_tc_kernel<D>),
                               static_cast<int>(C::kQSmem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(attn_bwd_dq_tc_kernel<D>, dim3(n_groups * BH), dim3(C::kThreads), C::kQSmem,
                   stream, tmQ, tmDO, tmK, tmV, static_cast<const bf16*>(a.o),
                   static_cast<const bf16*>(a.dout), a.lse, a.dsum, a.dq, a.B, a.S, a.Hq, a.Hkv,
                   G_log2, n_groups, a.causal, a.ld, a.dev_err);
    count_launches(1);
    if (e != cudaSuccess) return e;
  }
  // dkv pass: the query halves of a key group are cut into chunks of at most
  // L halves, L sized for about six waves of one CTA per SM (at least 16, so
  // a chunk's K / V load and atomic epilogue stay small beside its work)
  {
    const int n_kgroups = (a.S + C::kTiles * 128 - 1) / (C::kTiles * 128);
    const int64_t rows_all = static_cast<int64_t>(a.S) << G_log2;
    const int64_t halves_all = (rows_all + 63) >> 6;
    int64_t work = 0, longest = 0;
    for (int kg = 0; kg < n_kgroups; ++kg) {
      const int64_t u_first =
          a.causal ? ((static_cast<int64_t>(kg) * C::kTiles * 128) << G_log2) >> 6 : 0;
      work += halves_all - u_first;
      longest = std::max<int64_t>(longest, halves_all - u_first);
    }
    work *= BH;
    const int64_t waves6 = 6 * static_cast<int64_t>(sm_count());
    int64_t L = (work + waves6 - 1) / waves6;
    if (L < 16) L = 16;
    if (L > longest) L = longest;
    const int max_chunks = static_cast<int>((longest + L - 1) / L);
    const size_t kv_bytes = static_cast<size_t>(BH) * a.S * D * sizeof(float);
    cudaError_t e = cudaMemsetAsync(a.dk, 0, kv_bytes, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(a.dv, 0, kv_bytes, stream);
    if (e != cudaSuccess) return e;
    e = allow_smem(reinterpret_cast<const void*>(attn_bwd_dkv_tc_kernel<D>),
                   static_cast<int>(C::kKSmem));
    if (e != cudaSuccess) return e;
    e = launch_pdl(attn_bwd_dkv_tc_kernel<D>, dim3(n_kgroups * max_chunks * BH), dim3(C::kThreads),
                   C::kKSmem, stream, tmQh, tmDOh, tmK, tmV, static_cast<const float*>(a.lse),
                   static_cast<const float*>(a.dsum), a.dk, a.dv, a.B, a.S, a.Hkv, G_log2,
                   a.causal, a.ld, static_cast<int>(L), max_chunks, a.dev_err);
    count_launches(1);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

bool attn_bwd_tc_supported(int d, int G) {
  return (d == 32 || d == 64 || d == 128) && G >= 1 && G <= 64 && (G & (G - 1)) == 0;
}

cudaError_t launch_attn_bwd_tc(const AttnBwdTcArgs& a, cudaStream_t stream) {
  if (!attn_bwd_tc_supported(a.d, a.G) || (a.ld & 63) != 0 ||
      a.ld < (static_cast<int64_t>(a.S) * a.G + 63) / 64 * 64)
    return cudaErrorInvalidValue;
  switch (a.d) {
    case 32: return launch_bwd_tc<32>(a, stream);
    case 64: return launch_bwd_tc<64>(a, stream);
    case 128: return launch_bwd_tc<128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ccgqa
