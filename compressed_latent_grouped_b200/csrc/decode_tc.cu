// Decode attention on the 5th-generation tensor core (bf16): one query token
// per sequence against the latent KV cache ("Compressed Convolutional
// Attention", Probleemstelling 2; "Grouped Query Attention (GQA)", "Por qué
// GQA reduce la caché KV": decode is bound by reading the cache).
//
// One CTA = one (sequence, kv group, split).  It streams its split of the
// cache in 128-key chunks; every K/V byte is read from HBM once and serves all
// G query heads of the group.
//   warp 0     TMA producer: K and V chunks (128 keys, swizzled) through a ring
//   warp 1     TMEM owner; one thread issues the MMAs:
//                S^T = K_c Q^T     (M = 128 keys, N = 16: the G heads, zero
//                                   padded; two TMEM buffers, so the scores of
//                                   chunk c+1 are ready when chunk c is done)
//                O^T += V_c^T P^T  (d >= 64: M = d, N = 16, V read MN-major,
//                                   P^T a 16 x 128 tile)
//                O  += P_c V_c     (d = 32: M = 128, P rows 0..G-1 are the
//                                   heads, the other rows stay zero; N = d)
//   warps 2-5  softmax: thread k owns key k of the chunk and its G scores; one
//              barrier-OR tells whether any score passed the running max by
//              more than 2^8 (only then is the chunk max reduced and O
//              rescaled), exp2 once per (key, head), P written to shared memory.  Keys at
//              or past len + 1 are masked and their V rows zeroed (a stale cache
//              row may hold anything, and 0 * NaN is NaN in the MMA).
// Each split writes (max, sum, unnormalised output) per head; the last CTA of a
// (sequence, group) -- found with an atomic ticket, never by waiting -- merges
// the splits, and the last group of a sequence bumps len.  Every wait is
// bounded; no cluster multicast is used.
#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kDecTcThreads = 192;
constexpr int kChunk = 128;          // keys per MMA chunk
constexpr int kQRows = 16;           // N of the S^T MMA: heads of the group, zero padded
constexpr float kLog2eD = 1.4426950408889634f;
constexpr float kRescale = 8.0f;

template <int D>
struct DCfg {
  static constexpr int kPanelCols = (D == 32) ? 32 : 64;
  static constexpr int kPanels = D / kPanelCols;
  static constexpr uint32_t kRowBytes = kPanelCols * 2;
  static constexpr uint32_t kSwz = (D == 32) ? kSwizzle64B : kSwizzle128B;
  static constexpr uint32_t kSbo = 8 * kRowBytes;
  static constexpr uint32_t kPanelBytes = kChunk * kRowBytes;   // one panel of 128 keys
  static constexpr uint32_t kTileBytes = kChunk * D * 2;        // K or V chunk
  static constexpr int kStages = (D == 128) ? 2 : 3;   // d = 64: ~104 KB, two CTAs per SM
  static constexpr uint32_t kQPanelBytes = kQRows * kRowBytes;
  // d >= 64: O^T = V^T P^T with P^T [16 heads][128 keys]; d = 32: O = P V with
  // P [128 rows][128 keys] (M must be 64 or 128).
  static constexpr bool kT = D >= 64;
  static constexpr uint32_t kPRows = kT ? kQRows : 128;
  static constexpr uint32_t kPPanelBytes = kPRows * 128;       // 64 keys x 2 B per row
  static constexpr uint32_t kPBufBytes = 2 * kPPanelBytes;     // one P tile (two key panels)
  static constexpr uint32_t kPBytes = 2 * kPBufBytes;          // double-buffered across chunks
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffV = kOffK + kStages * kTileBytes;
  static constexpr uint32_t kOffP = kOffV + kStages * kTileBytes;
  static constexpr uint32_t kOffQ = kOffP + kPBytes;
  static constexpr uint32_t kOffBar = kOffQ + ((kPanels * kQPanelBytes + 1023) & ~1023u);
  static constexpr int kMaxIds = 512;                        // page ids staged per split
  static constexpr uint32_t kOffIds = kOffBar + 1024;        // after barriers | TMEM slot | red[2][4][16]
  static constexpr size_t kSmem = kOffIds + kMaxIds * 4 + 1024;
  static constexpr uint32_t kColS = 0, kColO = 32, kTmemCols = 64;   // S^T x2 | O^T or O
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int D>
__global__ void __launch_bounds__(kDecTcThreads, 1)
    decode_attn_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, const DecodeArgs<bf16> a) {
  pdl_enter();
  using C = DCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;                   // [kStages] K ring
  uint64_t* k_empty = k_full + C::kStages;   // [kStages] released when S of that chunk is done
  uint64_t* v_full = k_empty + C::kStages;   // [kStages] V ring
  uint64_t* v_empty = v_full + C::kStages;   // [kStages] released when PV of that chunk is done
  uint64_t* q_ready = v_empty + C::kStages;  // 128 arrivals: Q^T and zeroed P built
  uint64_t* s_full = q_ready + 1;            // [2] S^T buffers
  uint64_t* p_full = s_full + 2;             // [2] 128 arrivals: P of chunks using buffer 0 / 1
  uint64_t* o_done = p_full + 2;             // [2] PV of chunks using P buffer 0 / 1
  uint64_t* drain = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffBar + 256);
  float* red = reinterpret_cast<float*>(smem + C::kOffBar + 512);   // [2][4 warps][kQRows]
  __shared__ int abort_flag, last_flag;

  const int sp = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int G = a.G;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  const int L = __ldcg(a.len + b);
  const bool valid_b = L >= 0 && L < a.cap;
  const int n_keys = valid_b ? L + 1 : 0;
  const int k0 = sp * a.chunk;
  const int k1 = min(k0 + a.chunk, n_keys);
  const int n_ch = k1 > k0 ? (k1 - k0 + kChunk - 1) / kChunk : 0;
  const int bg = b * a.Hkv + g;

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(q_ready, 128);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 128);
    mbar_init(&p_full[1], 128);
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
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

  float m_run[kQRows], l_part[kQRows];   // softmax threads: per head running max, own partial sum
#pragma unroll
  for (int h = 0; h < kQRows; ++h) {
    m_run[h] = -INFINITY;
    l_part[h] = 0.f;
  }

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // One thread streams K and V through two rings, polling both without
    // blocking on either: a K slot frees as soon as the S of its chunk is
    // computed, well before the PV that frees the V slot, so the K loads run
    // ahead of the V loads.
    volatile int* abort_v = &abort_flag;
    if (a.pages.table == nullptr) {
      if (lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        int ck = 0, cv = 0;
        long long t_last = clock64();
        while (ck < n_ch || cv < n_ch) {
          bool progress = false;
          if (ck < n_ch && mbar_test(&k_empty[ck % C::kStages], ((ck / C::kStages) & 1) ^ 1)) {
            const int st = ck % C::kStages;
            mbar_arrive_expect_tx(&k_full[st], C::kTileBytes);
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p)
              tma_load_3d(smem + C::kOffK + st * C::kTileBytes + p * C::kPanelBytes, &tmK,
                          &k_full[st], p * C::kPanelCols, k0 + ck * kChunk, bg);
            ++ck;
            progress = true;
          }
          if (cv < n_ch && mbar_test(&v_empty[cv % C::kStages], ((cv / C::kStages) & 1) ^ 1)) {
            const int st = cv % C::kStages;
            mbar_arrive_expect_tx(&v_full[st], C::kTileBytes);
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p)
              tma_load_3d(smem + C::kOffV + st * C::kTileBytes + p * C::kPanelBytes, &tmV,
                          &v_full[st], p * C::kPanelCols, k0 + cv * kChunk, bg);
            ++cv;
            progress = true;
          }
          if (progress) {
            t_last = clock64();
          } else if (*abort_v || clock64() - t_last > kWaitLimitCycles) {
            if (!*abort_v) {
              *abort_v = 1;
              raise_dev_err(a.dev_err, CCGQA_DEVERR_TIMEOUT);
            }
            break;
          }
        }
      }
    } else {
      // Paged cache: a chunk is nb = 128 / bx boxes of bx = min(page, 128) rows,
      // each at (row in page, page * Hkv + g) of the pool.  The warp first
      // stages the split's page ids (box i of the split at ids[i]) in shared
      // memory, then lane 0 alone polls and issues as for a contiguous cache
      // (ids past the staged ones are read from global memory).  Boxes wholly
      // past the sequence are not loaded (their keys are masked and V rows
      // zeroed); a page id outside the pool becomes a coordinate past the
      // pool, which TMA fills with zeros.
      const int shift = a.pages.shift;
      const int bx = min(1 << shift, kChunk);
      const int nb = kChunk / bx;
      const int pool_z = a.pages.n_pages * a.Hkv;
      const int32_t* ptab = a.pages.table + static_cast<int64_t>(b) * a.pages.per_seq;
      int* ids = reinterpret_cast<int*>(smem + C::kOffIds);
      if (n_ch > 0) {
        const int n_ids = min((k1 - k0 + bx - 1) / bx, C::kMaxIds);
        for (int i = lane; i < n_ids; i += 32) ids[i] = __ldg(ptab + ((k0 + i * bx) >> shift));
      }
      __syncwarp();
      if (lane == 0) {
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
        auto load_chunk = [&](uint8_t* dst, const CUtensorMap* tm, uint64_t* bar, int c) {
          const int t0 = k0 + c * kChunk;
          const int nbox = min(nb, (k1 - t0 + bx - 1) / bx);
          mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbox * bx) * C::kRowBytes * C::kPanels);
          for (int j = 0; j < nbox; ++j) {
            const int i = c * nb + j;
            const int pg = i < C::kMaxIds ? ids[i] : __ldg(ptab + ((k0 + i * bx) >> shift));
            const bool ok_pg = pg >= 0 && pg < a.pages.n_pages;
            if (!ok_pg) raise_dev_err(a.dev_err, CCGQA_DEVERR_INDEX);
            const int row = (t0 + j * bx) & ((1 << shift) - 1);
#pragma unroll
            for (int p = 0; p < C::kPanels; ++p)
              tma_load_3d(dst + p * C::kPanelBytes + j * bx * C::kRowBytes, tm, bar,
                          p * C::kPanelCols, row, ok_pg ? pg * a.Hkv + g : pool_z);
          }
        };
        int ck = 0, cv = 0;
        long long t_last = clock64();
        while (ck < n_ch || cv < n_ch) {
          bool progress = false;
          if (ck < n_ch && mbar_test(&k_empty[ck % C::kStages], ((ck / C::kStages) & 1) ^ 1)) {
            const int st = ck % C::kStages;
            load_chunk(smem + C::kOffK + st * C::kTileBytes, &tmK, &k_full[st], ck);
            ++ck;
            progress = true;
          }
          if (cv < n_ch && mbar_test(&v_empty[cv % C::kStages], ((cv / C::kStages) & 1) ^ 1)) {
            const int st = cv % C::kStages;
            load_chunk(smem + C::kOffV + st * C::kTileBytes, &tmV, &v_full[st], cv);
            ++cv;
            progress = true;
          }
          if (progress) {
            t_last = clock64();
          } else if (*abort_v || clock64() - t_last > kWaitLimitCycles) {
            if (!*abort_v) {
              *abort_v = 1;
              raise_dev_err(a.dev_err, CCGQA_DEVERR_TIMEOUT);
            }
            break;
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // S(0) S(1) | PV(0) S(2) | PV(1) S(3) | ...   S(c+2) reuses the buffer of S(c),
    // which the softmax has read once it arrived on p_full(c).
    if (lane == 0 && n_ch > 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, kQRows, false);
      const uint32_t idesc_o = C::kT ? make_idesc_bf16(D, kQRows, false, true)
                                     : make_idesc_bf16(128, D, true);
      const uint32_t q_base = smem_addr(smem + C::kOffQ);
      const uint32_t p_base = smem_addr(smem + C::kOffP);
      auto issue_s = [&](int c) {
        const int st = c % C::kStages;
        const uint32_t k_base = smem_addr(smem + C::kOffK + st * C::kTileBytes);
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int p = (k * 16) / C::kPanelCols;
          const uint32_t off = ((k * 16) % C::kPanelCols) * 2;
          const uint64_t ad = make_smem_desc(k_base + p * C::kPanelBytes + off, 16, C::kSbo, C::kSwz);
          const uint64_t bd = make_smem_desc(q_base + p * C::kQPanelBytes + off, 16, C::kSbo, C::kSwz);
          mma_ss(tmem + C::kColS + (c & 1) * 16, ad, bd, idesc_s, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[c & 1]);
        mma_commit(&k_empty[st]);   // K slot free once this S is computed
      };
      auto issue_pv = [&](int c) {
        const int st = c % C::kStages;
        const uint32_t v_base = smem_addr(smem + C::kOffV + st * C::kTileBytes);
#pragma unroll
        for (int k = 0; k < kChunk / 16; ++k) {
          // V: MN-major (d contiguous), 16 keys = 16 rows of the swizzle width
          const uint64_t vd = make_smem_desc(v_base + k * 16 * C::kRowBytes, C::kPanelBytes,
                                             C::kSbo, C::kSwz);
          // P (or P^T): K-major over keys, two 64-key panels, 128B swizzle
          const uint64_t pd = make_smem_desc(p_base + (c & 1) * C::kPBufBytes +
                                                 (k >> 2) * C::kPPanelBytes + (k & 3) * 32,
                                             16, 1024, kSwizzle128B);
          if constexpr (C::kT)
            mma_ss(tmem + C::kColO, vd, pd, idesc_o, (c > 0 || k > 0) ? 1u : 0u);
          else
            mma_ss(tmem + C::kColO, pd, vd, idesc_o, (c > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(&o_done[c & 1]);
        mma_commit(&v_empty[st]);
      };
      bool ok = mbar_wait(q_ready, 0, &abort_flag, a.dev_err);
      for (int c = 0; ok && c < 2 && c < n_ch; ++c) {
        if (!mbar_wait(&k_full[c % C::kStages], (c / C::kStages) & 1, &abort_flag, a.dev_err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(c);
      }
      volatile int* abort_v = &abort_flag;
      for (int c = 0; ok && c < n_ch; ++c) {
        if (!mbar_wait(&p_full[c & 1], (c >> 1) & 1, &abort_flag, a.dev_err)) break;
        // PV(c) needs V(c); S(c+2) reuses the S buffer the softmax has just
        // released and needs K(c+2): issue whichever is ready first.
        bool pv_left = true, s_left = c + 2 < n_ch;
        const uint32_t vpar = (c / C::kStages) & 1, kpar = ((c + 2) / C::kStages) & 1;
        const long long t0c = clock64();
        while (pv_left || s_left) {
          if (pv_left && mbar_test(&v_full[c % C::kStages], vpar)) {
            tc_fence_after();
            issue_pv(c);
            pv_left = false;
          }
          if (s_left && mbar_test(&k_full[(c + 2) % C::kStages], kpar)) {
            tc_fence_after();
            issue_s(c + 2);
            s_left = false;
          }
          if ((pv_left || s_left) && (*abort_v || clock64() - t0c > kWaitLimitCycles)) {
            if (!*abort_v) {
              *abort_v = 1;
              raise_dev_err(a.dev_err, CCGQA_DEVERR_TIMEOUT);
            }
            ok = false;
            break;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int sw = warp - 2;                   // 0..3
    const int q4 = warp & 3;
    const int key = q4 * 32 + lane;            // row of the chunk == TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const int t128 = tid - 64;                 // 0..127 among the softmax threads
    uint8_t* ptile = smem + C::kOffP;
    // Q^T tile: rows 0..G-1 are this group's queries (bf16), the rest zero;
    // P / P^T tile: all zero (rows >= G stay zero for the whole CTA).
    for (int i = t128; i < static_cast<int>(C::kPBytes / 16); i += 128)
      reinterpret_cast<uint4*>(ptile)[i] = make_uint4(0, 0, 0, 0);
    {
      // all loads first, then the stores (one memory latency, not one per element)
      const float* qsrc = a.q_ws + (static_cast<int64_t>(b) * a.Hq + g * G) * D;
      constexpr int kPer = kQRows * D / 128;
      float qv[kPer];
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = t128 + u * 128, h = i / D;
        qv[u] = h < G ? __ldcg(qsrc + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kPer; ++u) {
        const int i = t128 + u * 128, h = i / D, e = i - h * D;
        const int p = e / C::kPanelCols, ec = e % C::kPanelCols;
        *reinterpret_cast<bf16*>(smem + C::kOffQ + p * C::kQPanelBytes +
                                 swz_offset(h, ec * 2, C::kRowBytes)) = __float2bfloat16_rn(qv[u]);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);
    const float scale = kLog2eD * rsqrtf(static_cast<float>(D));
    bool ok = true;
    for (int c = 0; c < n_ch; ++c) {
      if (!mbar_wait(&s_full[c & 1], (c >> 1) & 1, &abort_flag, a.dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[16];
      tmem_ld16(trow + C::kColS + (c & 1) * 16, sr);
      tmem_wait_ld();
      const int kk = k0 + c * kChunk + key;
      const bool kv = kk < k1;
      float sv[kQRows];
#pragma unroll
      for (int h = 0; h < kQRows; ++h) sv[h] = (kv && h < G) ? __uint_as_float(sr[h]) * scale : -INFINITY;
      // The running max per head only moves when some key of the chunk lies
      // more than kRescale above it; one barrier-OR over the 128 softmax
      // threads answers that, and only then is the chunk max formed (warp
      // shuffles, then the four warps' maxima through shared memory).
      bool over = false;
#pragma unroll
      for (int h = 0; h < kQRows; ++h) {
        if (h >= G) break;
        over |= sv[h] > m_run[h] + kRescale;   // also when m_run is still -inf
      }
      bool need_any = false;
      float factor[kQRows];
#pragma unroll
      for (int h = 0; h < kQRows; ++h) factor[h] = 1.f;
      if (named_barrier_or(1, 128, over)) {
        float* rb = red + (c & 1) * 4 * kQRows;   // double-buffered across chunks
#pragma unroll
        for (int h = 0; h < kQRows; ++h) {
          if (h >= G) break;
          float m = sv[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
          if (lane == 0) rb[sw * kQRows + h] = m;
        }
        named_barrier_sync(1, 128);
#pragma unroll
        for (int h = 0; h < kQRows; ++h) {
          if (h >= G) break;
          const float cm = fmaxf(fmaxf(rb[h], rb[kQRows + h]), fmaxf(rb[2 * kQRows + h], rb[3 * kQRows + h]));
          if (cm > m_run[h] + kRescale) {
            factor[h] = (m_run[h] == -INFINITY) ? 0.f : ex2(m_run[h] - cm);
            m_run[h] = cm;
            need_any = true;
            l_part[h] *= factor[h];
          }
        }
      }
      float p[kQRows];
#pragma unroll
      for (int h = 0; h < kQRows; ++h) {
        if (h >= G) break;
        p[h] = (m_run[h] == -INFINITY) ? 0.f : ex2(sv[h] - m_run[h]);
        l_part[h] += p[h];
      }
      // P buffer c&1 was last read by PV(c-2); a rescale needs O to hold PV(c-1)
      if (c >= 2) {
        if (!mbar_wait(&o_done[c & 1], ((c - 2) >> 1) & 1, &abort_flag, a.dev_err)) {
          ok = false;
          break;
        }
      }
      if (need_any && c >= 1) {
        if (!mbar_wait(&o_done[(c - 1) & 1], ((c - 1) >> 1) & 1, &abort_flag, a.dev_err)) {
          ok = false;
          break;
        }
      }
      tc_fence_after();
      if (need_any) {
        if constexpr (C::kT) {
          // O^T: TMEM lane = output channel, column h = head h
          uint32_t o[16];
          tmem_ld16(trow + C::kColO, o);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kQRows; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * factor[h]);
          tmem_st16(trow + C::kColO, o);
          tmem_wait_st();
        } else if (q4 == 0) {
          // O rows 0..G-1 live in TMEM lanes 0..G-1
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(trow + C::kColO + cc * 32, o);
            tmem_wait_ld();
            float f = 1.f;
#pragma unroll
            for (int h = 0; h < kQRows; ++h)
              if (lane == h) f = factor[h];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(trow + C::kColO + cc * 32, o);
          }
          tmem_wait_st();
        }
      }
      // P[h][key] into the K-major 128B-swizzled P tile (two 64-key panels)
#pragma unroll
      for (int h = 0; h < kQRows; ++h) {
        if (h >= G) break;
        *reinterpret_cast<bf16*>(ptile + (c & 1) * C::kPBufBytes + (key >> 6) * C::kPPanelBytes +
                                 swz_offset(h, (key & 63) * 2, 128)) = __float2bfloat16_rn(p[h]);
      }
      if (!kv && mbar_wait(&v_full[c % C::kStages], (c / C::kStages) & 1, &abort_flag, a.dev_err)) {
        // zero the V row of a key past the sequence (its P is zero, but 0 * NaN
        // is not) once the V chunk has landed
        uint8_t* vt = smem + C::kOffV + (c % C::kStages) * C::kTileBytes;
#pragma unroll
        for (int pn = 0; pn < C::kPanels; ++pn)
#pragma unroll
          for (int cb = 0; cb < static_cast<int>(C::kRowBytes); cb += 16)
            *reinterpret_cast<uint4*>(vt + pn * C::kPanelBytes + swz_offset(key, cb, C::kRowBytes)) =
                make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[c & 1]);
    }
    // ---- split partials: max and sum per head, unnormalised O rows
    // the last PV completes after every earlier one
    const bool have = ok && n_ch > 0 && !abort_flag &&
                      mbar_wait(&o_done[(n_ch - 1) & 1], ((n_ch - 1) >> 1) & 1, &abort_flag, a.dev_err);
    tc_fence_after();
    named_barrier_sync(1, 128);   // everyone is done reading red[] of the last chunk
#pragma unroll
    for (int h = 0; h < kQRows; ++h) {
      if (h >= G) break;
      float s = l_part[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      if (lane == 0) red[sw * kQRows + h] = s;
    }
    named_barrier_sync(1, 128);
    const int64_t pbase = (static_cast<int64_t>(bg) * a.splits + sp) * G;
    if (t128 < G) {
      const int h = t128;
      float mh = -INFINITY;
#pragma unroll
      for (int hh = 0; hh < kQRows; ++hh)
        if (hh == h) mh = m_run[hh];
      a.part_ml[(pbase + h) * 2] = have ? mh : -INFINITY;
      a.part_ml[(pbase + h) * 2 + 1] =
          have ? red[h] + red[kQRows + h] + red[2 * kQRows + h] + red[3 * kQRows + h] : 0.f;
    }
    if constexpr (C::kT) {
      // O^T row e (output channel) sits in lane (e % 16) + 32 (e / 16) for d = 64
      // (M = 64 layout) and in lane e for d = 128 (M = 128).
      uint32_t o[16];
      tmem_ld16(trow + C::kColO, o);
      tmem_wait_ld();
      const int e = (D == 64) ? q4 * 16 + lane : q4 * 32 + lane;
      if (D == 128 || lane < 16) {
#pragma unroll
        for (int h = 0; h < kQRows; ++h)
          if (h < G) a.part_o[(pbase + h) * D + e] = have ? __uint_as_float(o[h]) : 0.f;
      }
    } else if (q4 == 0) {
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t o[32];
        tmem_ld32(trow + C::kColO + cc * 32, o);
        tmem_wait_ld();
        if (lane < G) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            a.part_o[(pbase + lane) * D + cc * 32 + e] = have ? __uint_as_float(o[e]) : 0.f;
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

  // ---- the last CTA of (b, g) merges every split
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(a.tickets + bg, 1);
    last_flag = (prev == a.splits - 1);
  }
  __syncthreads();
  if (!last_flag) return;
  __threadfence();
  // Two passes, each with its loads in flight together: per head, the max over
  // the splits, then each split's weight 2^(m_s - M) and the total sum (one
  // thread per head, weights kept in the now idle K ring); then every output
  // element sums its splits' unnormalised rows with those weights.
  const int64_t gbase = static_cast<int64_t>(bg) * a.splits * G;
  float* wts = reinterpret_cast<float*>(smem + C::kOffK);   // [splits][G], then inv_l[G]
  float* inv_l = wts + a.splits * G;
  // (loops over splits run in blocks of 8 with the block's loads issued first,
  // so a block costs one memory latency)
  constexpr int kBlk = 8;
  if (tid < G) {
    const int h = tid;
    float M = -INFINITY;
    for (int s0 = 0; s0 < a.splits; s0 += kBlk) {
      float mv[kBlk];
#pragma unroll
      for (int u = 0; u < kBlk; ++u)
        mv[u] = s0 + u < a.splits
                    ? __ldcg(a.part_ml + (gbase + static_cast<int64_t>(s0 + u) * G + h) * 2)
                    : -INFINITY;
#pragma unroll
      for (int u = 0; u < kBlk; ++u) M = fmaxf(M, mv[u]);
    }
    float lsum = 0.f;
    for (int s0 = 0; s0 < a.splits; s0 += kBlk) {
      float mv[kBlk], lv[kBlk];
#pragma unroll
      for (int u = 0; u < kBlk; ++u) {
        const int64_t pi = gbase + static_cast<int64_t>(s0 + u) * G + h;
        mv[u] = s0 + u < a.splits ? __ldcg(a.part_ml + pi * 2) : -INFINITY;
        lv[u] = s0 + u < a.splits ? __ldcg(a.part_ml + pi * 2 + 1) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kBlk; ++u) {
        const float wgt = (mv[u] == -INFINITY) ? 0.f : ex2(mv[u] - M);
        lsum = fmaf(lv[u], wgt, lsum);
        if (s0 + u < a.splits) wts[(s0 + u) * G + h] = wgt;
      }
    }
    inv_l[h] = (valid_b && lsum > 0.f) ? 1.f / lsum : 0.f;
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kDecTcThreads) {
    const int h = idx / D, i = idx - h * D;
    float acc = 0.f;
    for (int s0 = 0; s0 < a.splits; s0 += kBlk) {
      float ov[kBlk];
#pragma unroll
      for (int u = 0; u < kBlk; ++u)
        ov[u] = s0 + u < a.splits
                    ? __ldcg(a.part_o + (gbase + static_cast<int64_t>(s0 + u) * G + h) * D + i)
                    : 0.f;
#pragma unroll
      for (int u = 0; u < kBlk; ++u)
        if (s0 + u < a.splits) acc = fmaf(ov[u], wts[(s0 + u) * G + h], acc);
    }
    a.out[static_cast<int64_t>(b) * a.Hq * D + (g * G + h) * D + i] = __float2bfloat16_rn(acc * inv_l[h]);
  }
  __syncthreads();
  if (tid == 0) {
    a.tickets[bg] = 0;
    __threadfence();
    const int prev = atomicAdd(a.tickets + a.B * a.Hkv + b, 1);
    if (prev == a.Hkv - 1) {
      a.tickets[a.B * a.Hkv + b] = 0;
      if (valid_b) a.len[b] = L + 1;
    }
  }
}

template <int D>
cudaError_t launch_tc(const DecodeArgs<bf16>& a, cudaStream_t stream) {
  using C = DCfg<D>;
  const CUtensorMapSwizzle swz = (D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tmK, tmV;
  // contiguous: [B Hkv][cap][d]; paged: [n_pages Hkv][page][d] with boxes of
  // min(page, 128) rows
  const bool paged = a.pages.table != nullptr;
  const uint64_t rows = paged ? (uint64_t{1} << a.pages.shift) : static_cast<uint64_t>(a.cap);
  const uint64_t planes = paged ? static_cast<uint64_t>(a.pages.n_pages) * a.Hkv
                                : static_cast<uint64_t>(a.B) * a.Hkv;
  const uint32_t box_rows = paged ? static_cast<uint32_t>(rows < kChunk ? rows : kChunk) : kChunk;
  const uint64_t dims[3] = {static_cast<uint64_t>(D), rows, planes};
  const uint64_t st[2] = {static_cast<uint64_t>(D) * 2, rows * D * 2};
  const uint32_t box[3] = {static_cast<uint32_t>(C::kPanelCols), box_rows, 1};
  if (!encode_tensor_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.cache_k, dims, st, box, swz) ||
      !encode_tensor_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.cache_v, dims, st, box, swz))
    return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(decode_attn_tc_kernel<D>),
                                       static_cast<int>(C::kSmem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.splits, a.Hkv, a.B);
  const cudaError_t el = launch_pdl(decode_attn_tc_kernel<D>, grid, dim3(kDecTcThreads),
                                    C::kSmem, stream, tmK, tmV, a);
  count_launches(1);
  return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_attn_tc(const DecodeArgs<bf16>& a, cudaStream_t stream) {
  if (a.G > kQRows) return cudaErrorInvalidValue;
  switch (a.d) {
    case 32: return launch_tc<32>(a, stream);
    case 64: return launch_tc<64>(a, stream);
    case 128: return launch_tc<128>(a, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace ccgqa
