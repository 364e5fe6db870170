// Causal grouped-query flash attention on the 5th-generation tensor core
// ("Compressed Convolutional Attention", section CCGQA: kv heads shared by a
// group of query heads inside the latent space; "Grouped Query Attention
// (GQA)", "Cómo funciona GQA").
//
// One CTA = one 128-row query tile of one kv group of one sequence.  The tile
// packs the group's G query heads: row r is position t0 + r / G, head
// g*G + r % G.  A 5-D TMA box gathers those rows straight from q[B, S, Hq, d],
// so one K/V tile load in shared memory serves all G query heads.
//
//   warp 0     TMA producer: Q once, then K/V tiles of 128 keys through a ring
//   warp 1     TMEM allocator; one elected thread issues every tcgen05.mma:
//                S_j = Q K_j^T   (SS, M=128 N=128, fp32 into TMEM, 2 buffers)
//                O  += P_j V_j   (SS, M=128 N=d, V read MN-major)
//   warps 2-5  softmax: each thread owns one row (TMEM lane), loads S_j with
//              tcgen05.ld, masks, keeps a running max / sum in registers,
//              writes bf16 P into a 128B-swizzled shared tile, rescales O in
//              TMEM when the running max grows by more than 2^8, and at the
//              end normalises O and stores it.
// The S double buffer lets the MMA of tile j+1 run under the softmax of tile j.
// No cluster multicast is used; every wait is bounded.
#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kAttnThreads = 192;
constexpr int kBlockM = 128, kBlockN = 128;
// exp(x) = exp2(x * log2(e)); scores are kept in the log2 domain.
constexpr float kLog2e = 1.4426950408889634f;
// The running max used for exp2 is only raised when it falls behind by more
// than this many doublings, so P <= 2^8 and O is rescaled rarely.
constexpr float kRescaleThreshold = 8.0f;

template <int D>
struct Cfg {
  static constexpr int kPanelCols = (D == 32) ? 32 : 64;      // elements per swizzle row
  static constexpr int kPanels = D / kPanelCols;
  static constexpr uint32_t kRowBytes = kPanelCols * 2;       // 64 or 128
  static constexpr uint32_t kSwz = (D == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;             // 8-row group stride
  static constexpr uint32_t kPanelBytes = 128 * kRowBytes;    // one panel of 128 rows
  static constexpr uint32_t kTileBytes = 128 * D * 2;         // Q / K / V tile
  static constexpr int kStages = (D == 128) ? 2 : 3;
  static constexpr uint32_t kPBytes = 128 * 128 * 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kTileBytes;
  static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
  static constexpr uint32_t kOffP = kOffV + kStages * kTileBytes;
  static constexpr uint32_t kOffBar = kOffP + kPBytes;
  static constexpr size_t kSmem = kOffBar + 256 + 1024;
  static constexpr uint32_t kTmemCols = 512;                  // S0 | S1 | O
  static constexpr uint32_t kColO = 256;
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                           const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, bf16* __restrict__ out,
                           int B, int S, int Hq, int Hkv, int G_log2, int n_qt, int causal,
                           int32_t* dev_err) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;                  // [kStages]
  uint64_t* kv_empty = kv_full + C::kStages;     // [kStages]
  uint64_t* s_full = kv_empty + C::kStages;      // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* drain = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = 1 << G_log2;
  const int BH = B * Hkv;
  const int qt = n_qt - 1 - static_cast<int>(blockIdx.x) / BH;  // longest tiles first
  const int bg = static_cast<int>(blockIdx.x) % BH;
  const int b = bg / Hkv, g = bg % Hkv;
  const int rows_pos = kBlockM >> G_log2;       // positions per tile
  const int t0 = qt * rows_pos;
  const int t_last = min(t0 + rows_pos - 1, S - 1);
  const int n_kv = causal ? (t_last / kBlockN + 1) : (S + kBlockN - 1) / kBlockN;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(pv_done, 1);
    mbar_init(drain, 1);
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
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, C::kTileBytes);
#pragma unroll
      for (int p = 0; p < C::kPanels; ++p)
        tma_load_5d(smem + C::kOffQ + p * C::kPanelBytes, &tmQ, q_full, p * C::kPanelCols, 0, g,
                    t0, b);
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
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(kBlockM, kBlockN, false);
      const uint32_t idesc_o = make_idesc_bf16(kBlockM, D, true);
      const uint32_t q_base = smem_addr(smem + C::kOffQ);
      const uint32_t p_base = smem_addr(smem + C::kOffP);
      auto issue_pv = [&](int jj) {
        const int st = jj % C::kStages;
        const uint32_t v_base = smem_addr(smem + C::kOffV + st * C::kTileBytes);
#pragma unroll
        for (int k = 0; k < kBlockN / 16; ++k) {
          // P: K-major, two 64-key panels of 128 rows x 128 B.
          const uint64_t ad = make_smem_desc(p_base + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024,
                                             kSwizzle128B);
          // V: MN-major (d contiguous); 16 keys = 16 rows of the swizzle width.
          const uint64_t bd = make_smem_desc(v_base + k * 16 * C::kRowBytes, C::kPanelBytes,
                                             C::kSbo, C::kSwz);
          mma_ss(tmem + C::kColO, ad, bd, idesc_o, (jj > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(pv_done);
        mma_commit(&kv_empty[st]);
      };
      bool ok = mbar_wait(q_full, 0, &abort_flag, dev_err);
      int j = 0;
      for (; ok && j < n_kv; ++j) {
        const int st = j % C::kStages;
        if (!mbar_wait(&kv_full[st], (j / C::kStages) & 1, &abort_flag, dev_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_base = smem_addr(smem + C::kOffK + st * C::kTileBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int p = (k * 16) / C::kPanelCols;
          const uint32_t off = p * C::kPanelBytes + ((k * 16) % C::kPanelCols) * 2;
          const uint64_t ad = make_smem_desc(q_base + off, 16, C::kSbo, C::kSwz);
          const uint64_t bd = make_smem_desc(k_base + off, 16, C::kSbo, C::kSwz);
          mma_ss(tmem + (j & 1) * kBlockN, ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[j & 1]);
        if (j > 0) {
          if (!mbar_wait(p_full, (j - 1) & 1, &abort_flag, dev_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_pv(j - 1);
        }
      }
      if (ok && n_kv > 0) {
        if (mbar_wait(p_full, (n_kv - 1) & 1, &abort_flag, dev_err)) {
          tc_fence_after();
          issue_pv(n_kv - 1);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;                 // tile row == TMEM lane
    const int t = t0 + (r >> G_log2);
    const int hl = r & (G - 1);
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const float scale = kLog2e * rsqrtf(static_cast<float>(D));
    float m_used = -INFINITY, l = 0.f;
    uint8_t* p_tile = smem + C::kOffP;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      if (!mbar_wait(&s_full[j & 1], (j >> 1) & 1, &abort_flag, dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        tmem_ld32(trow + (j & 1) * kBlockN + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_wait_ld();
      // keys s = j*128 + c are visible when c <= lim
      int lim = S - 1 - j * kBlockN;
      if (causal) lim = min(lim, t - j * kBlockN);
      float tmax = -INFINITY;
      float* sf = reinterpret_cast<float*>(sr);
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        const float v = (c <= lim) ? sf[c] * scale : -INFINITY;
        sf[c] = v;
        tmax = fmaxf(tmax, v);
      }
      const float m_new = fmaxf(m_used, tmax);
      bool need = false;
      float factor = 1.f;
      if (j == 0) {
        m_used = m_new;
      } else if (m_new > m_used + kRescaleThreshold) {
        factor = fast_exp2(m_used - m_new);
        l *= factor;
        m_used = m_new;
        need = true;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float p0 = fast_exp2(sf[2 * c] - mu);
        const float p1 = fast_exp2(sf[2 * c + 1] - mu);
        l += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[c] = *reinterpret_cast<uint32_t*>(&h2);
      }
      if (j > 0) {
        // O holds P_0..j-1 V: wait for the last PV before rescaling O or
        // overwriting the P tile it reads.
        if (!mbar_wait(pv_done, (j - 1) & 1, &abort_flag, dev_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(trow + C::kColO + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * factor);
            tmem_st32(trow + C::kColO + c * 32, o);
          }
          tmem_wait_st();
        }
      }
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        uint4 v = make_uint4(pk[cc * 4], pk[cc * 4 + 1], pk[cc * 4 + 2], pk[cc * 4 + 3]);
        *reinterpret_cast<uint4*>(p_tile + (cc >> 3) * 16384 + sw128_offset(r, cc & 7)) = v;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (ok && n_kv > 0 && mbar_wait(pv_done, (n_kv - 1) & 1, &abort_flag, dev_err)) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const bool store = t < S;
      bf16* dst = out + ((static_cast<int64_t>(b) * S + t) * Hq + g * G + hl) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(trow + C::kColO + c * 32, o);
        tmem_wait_ld();
        if (store) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 pkd;
            uint32_t* pw = reinterpret_cast<uint32_t*>(&pkd);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(o[v * 8 + 2 * e]) * inv_l,
                                                        __uint_as_float(o[v * 8 + 2 * e + 1]) * inv_l);
              pw[e] = *reinterpret_cast<uint32_t*>(&h2);
            }
            *reinterpret_cast<uint4*>(dst + c * 32 + v * 8) = pkd;
          }
        }
      }
    }
  }

  if (abort_flag && warp == 1 && lane == 0) {
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
  int G_log2 = 0;
  while ((1 << G_log2) < a.G) ++G_log2;
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
  cudaError_t e = cudaFuncSetAttribute(attn_prefill_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  const int n_qt = (a.S * a.G + kBlockM - 1) / kBlockM;
  const int grid = n_qt * a.B * a.Hkv;
  attn_prefill_tc_kernel<D><<<grid, kAttnThreads, C::kSmem, stream>>>(
      tmQ, tmK, tmV, static_cast<bf16*>(a.out), a.B, a.S, a.Hq, a.Hkv, G_log2, n_qt, a.causal,
      a.dev_err);
  count_launches(1);
  return cudaGetLastError();
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
