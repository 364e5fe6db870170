// Causal grouped-query flash attention on the 5th-generation tensor core
// ("Compressed Convolutional Attention", section CCGQA: kv heads shared by a
// group of query heads inside the latent space; "Grouped Query Attention
// (GQA)", "Cómo funciona GQA").
//
// Query rows are packed per kv group: row r of a tile is position
// t0 + r / G, head g*G + r % G, so a 5-D TMA box gathers a tile straight from
// q[B, S, Hq, d] and one K/V tile in shared memory serves all G query heads.
// A tile holds floor(128 / G) positions; when G does not divide 128 (the
// kPow2 = false instantiation) the last 128 mod G rows are zeroed once and
// never stored.
//
// One CTA owns T consecutive 128-row query tiles of one kv group (T = 3 at
// d = 32, else 2) and streams the K/V tiles they need once, as 128-key tiles
// split into two 64-key halves:
//   warp 0      TMA producer: the T query tiles once, then K/V tiles of 128
//               keys through a ring of shared-memory stages
//   warps 1..T  one thread each issues the tcgen05.mma of one query tile
//               (warp 1 also owns the TMEM allocation):
//                 S_X = Q_X K_h^T  (SS, M=128 N=64, fp32 accumulators in TMEM)
//                 O_X += P_X V_h   (TS: P read from TMEM, V from shared memory)
//               With one issuer per tile, waiting for one tile's PV never
//               delays the other tile's MMAs.
//   warps 4+4x..7+4x  softmax of tile x: one thread per
//               row (TMEM lane); tcgen05.ld of S, running max / sum in
//               registers, P written back to TMEM as bf16 pairs in the upper
//               half of its S buffer, O rescaled in TMEM on the rare half whose
//               partial sum shows the running max fell behind, normalised O
//               stored at the end.
// Each tile has two S buffers (one per 64-key half), so the S of the next half
// is computed while the softmax works on the current one and a softmax
// warpgroup never waits for the PV -> S round trip; the two warpgroups keep
// the exp unit and the FMA pipe busy while the tensor core runs their MMAs.
// TMEM: S/P of tile x at columns 128 x + {0, 64}, O_x at 128 T + x d.

// No cluster multicast is used; every wait is bounded.
#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kBlockM = 128, kBlockN = 128, kHalfN = 64;
constexpr float kLog2e = 1.4426950408889634f;
// The running max used for exp2 is only raised when a row's partial sum over
// a 64-key half exceeds this, so every P stays below 2^10 and O is rescaled
// rarely.
constexpr float kSumLimit = 1024.0f;

template <int D>
struct Cfg {
  static constexpr int kPanelCols = (D == 32) ? 32 : 64;      // elements per swizzle row
  static constexpr int kPanels = D / kPanelCols;
  static constexpr uint32_t kRowBytes = kPanelCols * 2;       // 64 or 128
  static constexpr uint32_t kSwz = (D == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;             // 8-row group stride
  static constexpr uint32_t kPanelBytes = 128 * kRowBytes;    // one panel of 128 rows
  static constexpr uint32_t kTileBytes = 128 * D * 2;         // one Q / K / V tile
  static constexpr int kStages = (D == 128) ? 2 : (D == 64 ? 3 : 4);
  // Query tiles per CTA: three where their S buffers and accumulators fit
  // in TMEM (3 x 128 + 3 x 32 columns at d = 32), else two.
  static constexpr int kTiles = (D == 32) ? 3 : 2;
  static constexpr int kSoftEvery = (D == 64) ? 3 : (D == 32 ? 5 : 4);
  static constexpr int kThreads = 128 + 128 * kTiles;   // 4 control warps + softmax
  static constexpr uint32_t kOffQ = 0;                        // Q_A, Q_B
  static constexpr uint32_t kOffK = kTiles * kTileBytes;
  static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
  static constexpr uint32_t kOffBar = kOffV + kStages * kTileBytes;
  static constexpr size_t kSmem = kOffBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static_assert(kTiles * 128 + kTiles * D <= 512, "S buffers and accumulators exceed TMEM");
  // S buffer h of tile x, its P (upper 32 columns: 64 keys as bf16 pairs), O_x
  __device__ static constexpr uint32_t col_s(int x, int h) { return x * 128 + h * 64; }
  __device__ static constexpr uint32_t col_p(int x, int h) { return x * 128 + h * 64 + 32; }
  __device__ static constexpr uint32_t col_o(int x) { return kTiles * 128 + x * D; }
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (one instruction for two lanes' worth of FMA-pipe work).
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

// 2^x on a pair, on the FMA pipe (packed fp32x2 steps), used for part of the
// probabilities so the exp unit and the FMA pipe share the work.  Cody-Waite
// style reduction x = n + f with
// n = round(x) and f in [-0.5, 0.5] (adding 1.5 * 2^23 leaves round(x) in the
// low mantissa bits), 2^f from a degree-3 polynomial fitted for this kernel
// (relative error below 8e-5, well under bf16's 2^-9), and 2^n added to the
// exponent field.  Inputs are clamped at -126 (the exponent field of p,
// 126 or 127, must stay positive after adding n), so -inf gives ~1e-38.  An
// input of kSoftArgMax or more would carry the exponent field past its top, so
// the caller tracks the largest input (one 3-input max per pair) and redoes
// the half against a raised running max when it gets there.
constexpr float kSoftArgMax = 127.0f;
__device__ __forceinline__ float2 soft_exp2x2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 big = make_float2(12582912.0f, 12582912.0f);
  const float2 t = fadd2(x, big);
  const float2 n = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);
  float2 p = ffma2(make_float2(0.05521968f, 0.05521968f), f, make_float2(0.24260941f, 0.24260941f));
  p = ffma2(p, f, make_float2(0.69325167f, 0.69325167f));
  p = ffma2(p, f, make_float2(0.99992800f, 0.99992800f));
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Pairs (c2 % Cfg<D>::kSoftEvery == 0) of each softmax row use the software
// exp2, so the FMA pipe takes part of the exponentials off the exp unit.
// Measured on B200: one pair in 3 is best at d = 64 (1.47 ms against 1.50 ms
// for 1 in 4 and 1.56 ms for 1 in 2 on S = 32768), one in 5 at d = 32 (174 us
// against 180 us for 1 in 4 and 177 us for 1 in 6 on 4 x 4096), one in 4 at
// d = 128.

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h2 = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h2);
}

template <int D, bool kPow2>
__global__ void __launch_bounds__(Cfg<D>::kThreads, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out,
                           int B, int S, int Hq, int Hkv, int G, int G_log2, int n_groups,
                           int causal, int32_t* dev_err, float* __restrict__ lse,
                           int64_t lse_ld) {
  pdl_enter();
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                  // [kStages]
  uint64_t* kv_empty = kv_full + C::kStages;     // [kStages]
  uint64_t* s_full = kv_empty + C::kStages;      // [tile][half]  S ready
  uint64_t* p_full = s_full + 2 * C::kTiles;     // [tile][half]  P written (128 arrivals)
  uint64_t* o_done = p_full + 2 * C::kTiles;     // [tile][half]  PV of that half complete
  uint64_t* drain = o_done + 2 * C::kTiles;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int BH = B * Hkv;
  const int grp = n_groups - 1 - static_cast<int>(blockIdx.x) / BH;  // longest first
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int b = bg / Hkv, g = bg % Hkv;
  const int pos_per_tile = kPow2 ? (kBlockM >> G_log2) : kBlockM / G;
  const int rows_used = pos_per_tile * G;     // rows of a tile the Q box fills
  const int t0 = grp * C::kTiles * pos_per_tile;
  const int t_last = min(t0 + C::kTiles * pos_per_tile - 1, S - 1);
  const int n_kv = causal ? (t_last / kBlockN + 1) : (S + kBlockN - 1) / kBlockN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], C::kTiles);   // released by every tile's last PV of the stage
    }
    for (int i = 0; i < 2 * C::kTiles; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&o_done[i], 1);
    }
    mbar_init(drain, C::kTiles);   // one commit from each MMA issuer
    abort_flag = 0;
    fence_barrier_init();
  }
  if (!kPow2 && rows_used < kBlockM) {
    // Rows the Q box does not fill (G does not divide 128): zero them so their
    // scores are finite; the MMA reads them through the async proxy.
    const int n16 = (kBlockM - rows_used) * C::kRowBytes / 16;
    for (int i = threadIdx.x; i < C::kTiles * C::kPanels * n16; i += blockDim.x) {
      const int tp = i / n16, w = i % n16;
      *reinterpret_cast<uint4*>(smem + C::kOffQ + tp * C::kPanelBytes + rows_used * C::kRowBytes +
                                w * 16) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
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
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, C::kTiles * rows_used * D * 2);
#pragma unroll
      for (int x = 0; x < C::kTiles; ++x)
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_5d(smem + C::kOffQ + x * C::kTileBytes + p * C::kPanelBytes, &tmQ, q_full,
                      p * C::kPanelCols, 0, g, t0 + x * pos_per_tile, b);
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % C::kStages;
        const uint32_t ph = (j / C::kStages) & 1;
        if (!mbar_wait(&kv_empty[st], ph ^ 1, &abort_flag, dev_err)) break;
        mbar_arrive_expect_tx(&kv_full[st], 2 * C::kTileBytes);
#pragma unroll
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_3d(smem + C::kOffK + st * C::kTileBytes + p * C::kPanelBytes, &tmK,
                      &kv_full[st], p * C::kPanelCols, j * kBlockN, bg);
          tma_load_3d(smem + C::kOffV + st * C::kTileBytes + p * C::kPanelBytes, &tmV,
                      &kv_full[st], p * C::kPanelCols, j * kBlockN, bg);
        }
      }
    }
  } else if (warp >= 1 && warp <= C::kTiles) {
    // ------------------------------------------------------------ MMA issuers
    // Tile x = warp - 1.  Per K/V tile j and half h: PV_x(j,h), then
    // S_x(j+1,h) into the buffer P_x(j,h) was read from (after that PV
    // completes); the softmax is meanwhile busy with the other half.
    if (lane == 0) {
      const int x = warp - 1;
      const uint32_t idesc_s = make_idesc_bf16(kBlockM, kHalfN, false);
      const uint32_t idesc_o = make_idesc_bf16(kBlockM, D, true);
      const uint32_t q_base = smem_addr(smem + C::kOffQ) + x * C::kTileBytes;
      auto issue_s = [&](int jj, int h) {
        const int st = jj % C::kStages;
        const uint32_t k_base =
            smem_addr(smem + C::kOffK + st * C::kTileBytes) + h * kHalfN * C::kRowBytes;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int p = (k * 16) / C::kPanelCols;
          const uint32_t off = p * C::kPanelBytes + ((k * 16) % C::kPanelCols) * 2;
          const uint64_t ad = make_smem_desc(q_base + off, 16, C::kSbo, C::kSwz);
          const uint64_t bd = make_smem_desc(k_base + off, 16, C::kSbo, C::kSwz);
          mma_ss(tmem + C::col_s(x, h), ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[x * 2 + h]);
      };
      auto issue_pv = [&](int jj, int h) {
        const int st = jj % C::kStages;
        const uint32_t v_base =
            smem_addr(smem + C::kOffV + st * C::kTileBytes) + h * kHalfN * C::kRowBytes;
#pragma unroll
        for (int k = 0; k < kHalfN / 16; ++k) {
          // V: MN-major (d contiguous); 16 keys = 16 rows of the swizzle width.
          const uint64_t bd = make_smem_desc(v_base + k * 16 * C::kRowBytes, C::kPanelBytes,
                                             C::kSbo, C::kSwz);
          // P: 16 keys per K step = 8 TMEM columns of bf16 pairs.
          mma_ts(tmem + C::col_o(x), tmem + C::col_p(x, h) + k * 8, bd, idesc_o,
                 (jj > 0 || h > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[x * 2 + h]);
      };
      bool ok = mbar_wait(q_full, 0, &abort_flag, dev_err) &&
                mbar_wait(&kv_full[0], 0, &abort_flag, dev_err);
      if (ok && n_kv > 0) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(0, 1);
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const bool more = j + 1 < n_kv;
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(&p_full[x * 2 + h], j & 1, &abort_flag, dev_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(j, h);
          if (h == 1) mma_commit(&kv_empty[j % C::kStages]);
          if (more) {
            if (h == 0 && !mbar_wait(&kv_full[(j + 1) % C::kStages], ((j + 1) / C::kStages) & 1,
                                     &abort_flag, dev_err)) {
              ok = false;
              break;
            }
            // S(j+1,h) overwrites the S buffer that holds P(j,h): PV(j,h) first
            if (!mbar_wait(&o_done[x * 2 + h], j & 1, &abort_flag, dev_err)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_s(j + 1, h);
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int x = (warp - 4) >> 2;                // query tile of this warpgroup
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // tile row == TMEM lane
    const int t = t0 + x * pos_per_tile + (kPow2 ? (r >> G_log2) : r / G);
    const int hl = kPow2 ? (r & (G - 1)) : r % G;
    const bool row_ok = kPow2 || r < rows_used;   // a row the Q box filled
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float scale = kLog2e * rsqrtf(static_cast<float>(D));
    const float2 scale2 = make_float2(scale, scale);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; ok && j < n_kv; ++j) {
      for (int h = 0; h < 2; ++h) {
        const int sb = x * 2 + h;
        if (!mbar_wait(&s_full[sb], j & 1, &abort_flag, dev_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // keys j*128 + h*64 + c are visible when c <= lim
        const int kb = j * kBlockN + h * kHalfN;
        int lim = S - 1 - kb;
        if (causal) lim = min(lim, t - kb);
        const bool full_half = __all_sync(0xffffffffu, lim >= kHalfN - 1);
        auto load_s = [&](float (&sv)[64]) {
          tmem_ld32(trow + C::col_s(x, h), *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
          tmem_ld32(trow + C::col_s(x, h) + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
          tmem_wait_ld();
          if (!full_half) {
#pragma unroll
            for (int c = 0; c < 64; ++c) sv[c] = (c <= lim) ? sv[c] : -INFINITY;
          }
        };
        auto row_max = [&](const float (&sv)[64]) {
          float mx[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = sv[k];
#pragma unroll
          for (int c = 8; c < 64; ++c) mx[c & 7] = fmaxf(mx[c & 7], sv[c]);
#pragma unroll
          for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], mx[k + 4]);
          return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * scale;
        };
        uint32_t pk[32];
        // p = 2^(s * scale - m_used) as bf16 pairs; returns the row's sum of p,
        // or +inf when an argument of the software exp2 passed its range (the
        // overflow the exp unit shows as inf): either way the half is redone
        auto exp_pass = [&](const float (&sv)[64]) {
          const float2 negm2 = make_float2(-m_used, -m_used);
          const float2* s2 = reinterpret_cast<const float2*>(sv);
          float2 lsum[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                            make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          float soft_max = -INFINITY;
#pragma unroll
          for (int c2 = 0; c2 < 32; ++c2) {
            const float2 arg = ffma2(s2[c2], scale2, negm2);
            float2 p;
            if ((c2 % C::kSoftEvery) == 0) {
              soft_max = fmax3(soft_max, arg.x, arg.y);
              p = soft_exp2x2(arg);
            } else {
              p.x = fast_exp2(arg.x);
              p.y = fast_exp2(arg.y);
            }
            lsum[c2 & 3] = fadd2(lsum[c2 & 3], p);
            pk[c2] = pack_bf16x2(p.x, p.y);
          }
          const float2 a2 = fadd2(fadd2(lsum[0], lsum[1]), fadd2(lsum[2], lsum[3]));
          return soft_max < kSoftArgMax ? a2.x + a2.y : INFINITY;
        };
        // The first half sets the running max (key 0 is visible to every
        // row, so it is finite).  Later halves exponentiate against the
        // running max as it stands and look only at the row's partial sum:
        // while it stays within kSumLimit every p is below it.  A row whose
        // sum overshoots (some p > kSumLimit / 64, so its max lies above the
        // running max by more than log2(kSumLimit / 64)) reloads S from TMEM,
        // which still holds it, raises the running max to the half's max and
        // redoes the half.
        float part;
        {
          float sv[64];
          load_s(sv);
          if (j == 0 && h == 0) m_used = row_max(sv);
          part = exp_pass(sv);
        }
        const bool redo = !(part <= kSumLimit);
        bool need = false;
        float factor = 1.f;
        if (__any_sync(0xffffffffu, redo)) {
          float sv[64];
          load_s(sv);   // warp-wide
          if (redo) {
            const float m_new = row_max(sv);
            factor = fast_exp2(m_used - m_new);
            l *= factor;
            m_used = m_new;
            need = true;
            part = exp_pass(sv);
          }
        }
        l += part;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold every earlier half: wait for the previous PV of this tile.
          const int pb = x * 2 + (1 - h);
          const uint32_t pph = (h == 1 ? j : j - 1) & 1;
          if (!mbar_wait(&o_done[pb], pph, &abort_flag, dev_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(trow + C::col_o(x) + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(trow + C::col_o(x) + c * 32, o);
          }
        }
        tmem_st32(trow + C::col_p(x, h), pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[sb]);
      }
    }
    // the last PV of this tile (half 1 of tile n_kv-1) completes after all others
    if (ok && n_kv > 0 && mbar_wait(&o_done[x * 2 + 1], (n_kv - 1) & 1, &abort_flag, dev_err)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = row_ok && t < S;
      if (lse != nullptr && store)
        lse[static_cast<int64_t>(bg) * lse_ld + static_cast<int64_t>(t) * G + hl] = -(m_used + log2f(l));
      bf16* dst = out + ((static_cast<int64_t>(b) * S + t) * Hq + g * G + hl) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(trow + C::col_o(x) + c * 32, o);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pkd;
            pkd.x = pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * inv_l, __uint_as_float(o[v * 8 + 1]) * inv_l);
            pkd.y = pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * inv_l, __uint_as_float(o[v * 8 + 3]) * inv_l);
            pkd.z = pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * inv_l, __uint_as_float(o[v * 8 + 5]) * inv_l);
            pkd.w = pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * inv_l, __uint_as_float(o[v * 8 + 7]) * inv_l);
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = pkd;
          }
        }
      }
    }
  }

  if (abort_flag && warp >= 1 && warp <= C::kTiles && lane == 0) {
    // Do not release TMEM while an MMA of either issuer might still write it.
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

template <int D>
cudaError_t launch_d(const AttnArgs& a, cudaStream_t stream) {
  using C = Cfg<D>;
  const CUtensorMapSwizzle swz =
      (D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tmQ, tmK, tmV;
  {
    // q[B, S, Hq, d] viewed as (d, G, Hkv, S, B): a box (panel, G, 1, 128/G, 1)
    // lands as 128 rows ordered (position, head-in-group).
    const uint64_t dims[5] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.G),
                              static_cast<uint64_t>(a.Hkv), static_cast<uint64_t>(a.S),
                              static_cast<uint64_t>(a.B)};
    const uint64_t st[4] = {static_cast<uint64_t>(D) * 2, static_cast<uint64_t>(a.G) * D * 2,
                            static_cast<uint64_t>(a.Hq) * D * 2,
                            static_cast<uint64_t>(a.S) * a.Hq * D * 2};
    const uint32_t box[5] = {static_cast<uint32_t>(C::kPanelCols), static_cast<uint32_t>(a.G), 1,
                             static_cast<uint32_t>(kBlockM / a.G), 1};
    if (!encode_tensor_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, a.q, dims, st, box, swz))
      return cudaErrorInvalidValue;
  }
  {
    // k/v[B, Hkv, cap, d] viewed as (d, S, B*Hkv): keys past S read as zero.
    const uint64_t dims[3] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.S),
                              static_cast<uint64_t>(a.B) * a.Hkv};
    const uint64_t st[2] = {static_cast<uint64_t>(D) * 2,
                            static_cast<uint64_t>(a.kv_cap) * D * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(C::kPanelCols), kBlockN, 1};
    if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.k, dims, st, box, swz) ||
        !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.v, dims, st, box, swz))
      return cudaErrorInvalidValue;
  }
  if (a.G < 1 || a.G > kBlockM) return cudaErrorInvalidValue;
  const int pos_per_cta = C::kTiles * (kBlockM / a.G);
  const int n_groups = (a.S + pos_per_cta - 1) / pos_per_cta;
  const int grid = n_groups * a.B * a.Hkv;
  int G_log2 = 0;
  while ((1 << G_log2) < a.G) ++G_log2;
  const bool pow2 = (1 << G_log2) == a.G;
  auto kernel = pow2 ? attn_prefill_tc_kernel<D, true> : attn_prefill_tc_kernel<D, false>;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kernel), static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const cudaError_t el = launch_pdl(kernel, dim3(grid), dim3(C::kThreads), C::kSmem, stream, tmQ,
                                    tmK, tmV, static_cast<bf16*>(a.out), a.B, a.S, a.Hq, a.Hkv,
                                    a.G, G_log2, n_groups, a.causal, a.dev_err, a.lse,
                                    a.lse_ld);
  count_launches(1);
  return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_prefill_tc(const AttnArgs& a, cudaStream_t stream) {
  switch (a.d) {
    case 32: return launch_d<32>(a, stream);
    case 64: return launch_d<64>(a, stream);
    case 128: return launch_d<128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ccgqa
