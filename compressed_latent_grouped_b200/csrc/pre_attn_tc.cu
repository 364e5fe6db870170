// Fused pre-attention with the per-head channel mix on the 5th-generation
// tensor core (bf16 heads of dim 32 or 64): causal sequence conv, channel mix,
// QK-mean, RoPE and value-shift ("Compressed Convolutional Attention",
// Methodologie items 2-4; the mix is a d x d product per position and head,
// i.e. a [positions x d] by [d x d] contraction).
//
// One CTA owns 128 consecutive positions of one kv group (its G query heads,
// its key head and its value head) of one sequence:
//   1. one thread issues the copies into shared memory: per head a TMA box of
//      the rows [t0 - 3, t0 + 128) of its d columns of q~ | k~ (rows outside
//      the sequence arrive as zeros; 64B / 128B swizzled rows), the G + 1 mix
//      weights W_h [d_out, d_in] as TMA tiles (straight into the swizzled
//      K-major layout of a UMMA B operand) and the conv taps as two bulk
//      copies, completing on one mbarrier per head in the order the heads use
//      them; meanwhile each thread loads its value-shift rows into registers
//      and forms the cos/sin of its own rotary pairs (angle t theta_i reduced
//      modulo one turn exactly in 64-bit fixed point);
//   2. per head h (G query heads, then the key head):
//        conv   one thread per (position, 16-byte channel chunk): u = sum_k
//               w[c, k] z[t - k, c] in fp32, split as u = hi + lo with hi, lo
//               bf16 and both written as the A operands [128 x d] of the MMA;
//        mix    one thread issues Y_h = U_hi W_h^T + U_lo W_h^T (M = 128, N = d,
//               fp32 accumulators in TMEM, two buffers), so the product keeps
//               fp32 accuracy (u - hi - lo is below 2^-16 |u|);
//        epilogue  thread = (position row = TMEM lane, half of the rotary pairs):
//               tcgen05.ld of Y_h, QK-mean from the staged pre-conv rows, RoPE on
//               the pairs (i, i + d/2) it holds, bf16 store.
//      The epilogue of head h - 1 runs while the tensor core computes head h.
//   3. value-shift: the rows loaded in step 1 are stored (bit-exact copies).
//   4. the CTA holding the last position writes the decode state.
// At d = 32 three CTAs fit on an SM (about 74 KB of shared memory each).
// Every wait is bounded; no cluster multicast is used.
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kPtThreads = 256;
constexpr int kPtTT = 128;     // positions per CTA == MMA M == TMEM lanes
constexpr int kPtHalo = 3;     // the conv reaches back K - 1 <= 3 rows

struct PtLayout {
  uint32_t u_bytes, w_bytes;   // one A tile (hi or lo), one head's B tile
  uint32_t zh_bytes;           // one head's staged rows (131 of d columns), 1024-aligned
  uint32_t off_u, off_w, off_z, off_ws, off_bar, bytes;
};

// Byte layout of the dynamic shared memory (from a 1024-byte aligned base).
__host__ __device__ inline PtLayout pt_layout(int d, int G) {
  PtLayout L;
  const uint32_t row = static_cast<uint32_t>(d) * 2;
  L.u_bytes = kPtTT * row;
  L.w_bytes = static_cast<uint32_t>(d) * row;
  L.zh_bytes = ((kPtTT + kPtHalo) * row + 1023u) & ~1023u;
  // U_hi | U_lo; before the first conv the same bytes hold the raw conv taps
  const uint32_t tr_bytes = (static_cast<uint32_t>(G + 1) * d * 4 * 2 + 15u) & ~15u;
  L.off_u = 0;
  L.off_w = 2 * L.u_bytes > tr_bytes ? 2 * L.u_bytes : tr_bytes;   // W_h, h = 0..G
  L.off_z = L.off_w + (G + 1) * L.w_bytes;          // head h's rows: off_z + h zh_bytes
  L.off_ws = L.off_z + (G + 1) * L.zh_bytes;
  L.off_bar = L.off_ws + static_cast<uint32_t>(G + 1) * d * 8;      // [(G+1) d][4] bf16
  L.bytes = L.off_bar + 8 * (G + 4) + 16 + 1024;    // barriers, TMEM slot, alignment slack
  return L;
}

// d = a * b + c for bf16 a, b and fp32 c, d in one instruction: the product
// of two bf16 values is exact in fp32, so this equals fmaf(float(a), float(b), c)
// and needs no conversion of a and b.
__device__ __forceinline__ float fma_bf16(uint16_t a, uint16_t b, float c) {
  float d;
  asm("fma.rn.f32.bf16 %0, %1, %2, %3;" : "=f"(d) : "h"(a), "h"(b), "f"(c));
  return d;
}
// d = a + c for bf16 a and fp32 c, d
__device__ __forceinline__ float add_bf16(uint16_t a, float c) {
  float d;
  asm("add.rn.f32.bf16 %0, %1, %2;" : "=f"(d) : "h"(a), "f"(c));
  return d;
}
// the two bf16 halves of a 32-bit word (low half = lower channel)
__device__ __forceinline__ void halves(uint32_t v, uint16_t& lo, uint16_t& hi) {
  asm("mov.b32 {%0, %1}, %2;" : "=h"(lo), "=h"(hi) : "r"(v));
}
constexpr uint16_t kBf16MinusOne = 0xBF80, kBf16Half = 0x3F00;

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// d = 32: three CTAs per SM (about 74 KB of shared memory and at most 85
// registers a thread each); d = 64: one.
template <int D>
__global__ void __launch_bounds__(kPtThreads, (D == 32) ? 3 : 1)
    pre_attn_tc_kernel(const __grid_constant__ CUtensorMap tmZ,
                       const __grid_constant__ CUtensorMap tmWq,
                       const __grid_constant__ CUtensorMap tmWk,
                       const __grid_constant__ PreAttnArgs<bf16> a) {
  pdl_enter();
  constexpr uint32_t kRowBytes = D * 2;                 // 64: 64B swizzle, 128: 128B swizzle
  constexpr uint32_t kSwz = (D == 32) ? kSwizzle64B : kSwizzle128B;
  constexpr uint32_t kSbo = 8 * kRowBytes;
  constexpr int NCH = D / 8;                            // 16-byte chunks per row
  constexpr int Q4 = D / 4;                             // rotary pairs per epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = a.G, S = a.S, K = a.K;
  const PtLayout L = pt_layout(D, G);
  const int NH = G + 1, QC = G * D;
  const int b = blockIdx.z, g = blockIdx.y, t0 = blockIdx.x * kPtTT;
  const int tid = threadIdx.x, warp = tid >> 5;
  uint8_t* z = smem + L.off_z;                           // head h: z + h zh_bytes
  uint2* ws = reinterpret_cast<uint2*>(smem + L.off_ws);   // taps of a channel: 4 bf16
  bf16* tr = reinterpret_cast<bf16*>(smem + L.off_u);   // raw taps, until the first conv
  uint64_t* mma_done = reinterpret_cast<uint64_t*>(smem + L.off_bar);   // [2]
  uint64_t* drain = mma_done + 2;
  uint64_t* ld_bar = drain + 1;       // [G]: 0 = taps, W, key head, query head 0; h = query head h
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ld_bar + G);
  __shared__ int abort_flag;

  const int64_t ld = a.src_ld;
  const bf16* src_b = a.src + static_cast<int64_t>(b) * S * ld;
  const int qcol0 = g * QC;
  const int kcol0 = a.Hq * D + g * D;
  const int vcol0 = (a.Hq + a.Hkv) * D + g * D;

  if (tid == 0) {
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    mbar_init(drain, 1);
    for (int h = 0; h < G; ++h) mbar_init(&ld_bar[h], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 2 * D);
    tmem_relinquish();
  }
  // barriers, abort flag and TMEM address visible before any thread uses them
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // 1. staging: one thread issues every copy (z boxes are 131 rows x d columns
  // of the [B][S][cols] tensor; head slot h < G is query head h, slot G the key
  // head; rows before position 0 and past S are zero-filled by the TMA unit)
  if (tid == 0) {
    prefetch_tensormap(&tmZ);
    prefetch_tensormap(&tmWq);
    prefetch_tensormap(&tmWk);
    const uint32_t zbox = (kPtTT + kPtHalo) * kRowBytes;
    const uint32_t tq = static_cast<uint32_t>(G) * D * K * 2, tk = static_cast<uint32_t>(D) * K * 2;
    mbar_arrive_expect_tx(&ld_bar[0], tq + tk + NH * L.w_bytes + 2 * zbox);
    bulk_load(tr, a.wq_seq + static_cast<int64_t>(g) * G * D * K, tq, &ld_bar[0]);
    bulk_load(reinterpret_cast<uint8_t*>(tr) + tq, a.wk_seq + static_cast<int64_t>(g) * D * K, tk,
              &ld_bar[0]);
    for (int h = 0; h < G; ++h)
      tma_load_2d(smem + L.off_w + h * L.w_bytes, &tmWq, &ld_bar[0], 0, (g * G + h) * D);
    tma_load_2d(smem + L.off_w + G * L.w_bytes, &tmWk, &ld_bar[0], 0, g * D);
    tma_load_3d(z + G * L.zh_bytes, &tmZ, &ld_bar[0], kcol0, t0 - kPtHalo, b);
    tma_load_3d(z, &tmZ, &ld_bar[0], qcol0, t0 - kPtHalo, b);
    for (int h = 1; h < G; ++h) {
      mbar_arrive_expect_tx(&ld_bar[h], zbox);
      tma_load_3d(z + h * L.zh_bytes, &tmZ, &ld_bar[h], qcol0 + h * D, t0 - kPtHalo, b);
    }
  }
  // value-shift rows straight into registers (stored at the end of the kernel):
  // v[t, :d/2] = v~[t, :d/2], v[t, d/2:] = v~[t-1, d/2:], zero before position 0
  // (whole-head reading: every channel of the group's kv head from t-1 when
  // the head is one of the last floor(Hkv/2))
  const bool shift_head = a.value_shift == 2 && g >= a.Hkv - a.Hkv / 2;
  constexpr int kVPer = kPtTT * NCH / kPtThreads;
  uint4 vreg[kVPer];
#pragma unroll
  for (int q = 0; q < kVPer; ++q) {
    const int idx = tid + q * kPtThreads;
    const int tl = idx / NCH, i = (idx % NCH) * 8;
    const int tv = t0 + tl;
    const int row = ((a.value_shift == 1 && i >= D / 2) || shift_head) ? tv - 1 : tv;
    vreg[q] = make_uint4(0, 0, 0, 0);
    if (tv < S && row >= 0)
      vreg[q] = *reinterpret_cast<const uint4*>(src_b + static_cast<int64_t>(row) * ld + vcol0 + i);
  }
  // RoPE of this thread's epilogue pairs (row tid % 128, pairs of half tid / 128)
  // while the copies fly: (cos, sin) of t * theta_i, the angle taken modulo one
  // turn exactly in 64-bit fixed point, then |2 pi f| <= pi.
  float rc[Q4], rs[Q4];
  {
    const int tp = t0 + (tid & (kPtTT - 1)), ip = (tid >> 7) * Q4;
#pragma unroll
    for (int e = 0; e < Q4; ++e) {
      rc[e] = 1.f;
      rs[e] = 0.f;
      if (a.rope_on) {
        const uint64_t ph = static_cast<uint64_t>(tp) * a.rope_frac[ip + e];
        const float f = static_cast<float>(static_cast<int64_t>(ph)) * 5.42101086242752217e-20f;
        __sincosf(6.28318530717958648f * f, &rs[e], &rc[e]);
      }
    }
  }
  bool ok = mbar_wait(&ld_bar[0], 0, &abort_flag, a.dev_err);   // taps, W, key head, query head 0
  // conv taps as bf16 [channel][4], zero past K
  for (int hc = tid; hc < NH * D; hc += kPtThreads) {
    uint16_t w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w4[k] = k < K ? __bfloat16_as_ushort(tr[hc * K + k]) : static_cast<uint16_t>(0);
    ws[hc] = make_uint2(w4[0] | (static_cast<uint32_t>(w4[1]) << 16),
                        w4[2] | (static_cast<uint32_t>(w4[3]) << 16));
  }
  __syncthreads();   // padded taps ready

  // 2. per head
  const int r = tid & (kPtTT - 1);         // position row == TMEM lane
  const int part = tid >> 7;               // conv chunks j = part (mod 2); pairs of half `part`
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t u_hi = smem_addr(smem + L.off_u);
  const uint32_t u_lo = u_hi + L.u_bytes;
  const uint32_t w_base = smem_addr(smem + L.off_w);
  const uint32_t idesc = make_idesc_bf16(kPtTT, D, false);
  const int t = t0 + r;
  // 16 bytes at channel chunk c of head slot h, staged row rr (swizzled rows)
  auto zchunk = [&](int h, int rr, int c) -> const uint4* {
    return reinterpret_cast<const uint4*>(z + h * L.zh_bytes + swz_offset(rr, c * 16, kRowBytes));
  };

  // conv of head hh for chunks j = P, P + 2, ... of row r (P: compile-time part):
  // u = sum_k w[c, k] z[t - k, c] by fp32 FMAs straight from the bf16 operands
  // (taps in order k = 0..3, as exact products), then u = hi + lo in bf16
  auto conv_part = [&](int hh, auto part_c) {
    constexpr int P = decltype(part_c)::value;
#pragma unroll
    for (int j = P; j < NCH; j += 2) {
      const uint4* tw = reinterpret_cast<const uint4*>(ws + hh * D + j * 8);   // 2 channels each
      uint4 t4[4], zz[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) t4[q] = tw[q];
#pragma unroll
      for (int k = 0; k < 4; ++k) zz[k] = *zchunk(hh, r + kPtHalo - k, j);
      float acc[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint4& tq = t4[e >> 1];
        uint16_t w[4], zv[4];
        halves((e & 1) ? tq.z : tq.x, w[0], w[1]);
        halves((e & 1) ? tq.w : tq.y, w[2], w[3]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t* zw = reinterpret_cast<const uint32_t*>(&zz[k]);
          uint16_t lo, hi;
          halves(zw[e >> 1], lo, hi);
          zv[k] = (e & 1) ? hi : lo;
        }
        float a = fma_bf16(zv[0], w[0], 0.f);
#pragma unroll
        for (int k = 1; k < 4; ++k) a = fma_bf16(zv[k], w[k], a);
        acc[e] = a;
      }
      uint4 hi4, lo4;
      uint32_t* hp = reinterpret_cast<uint32_t*>(&hi4);
      uint32_t* lp = reinterpret_cast<uint32_t*>(&lo4);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        hp[e] = pack2(acc[2 * e], acc[2 * e + 1]);
        uint16_t h0, h1;
        halves(hp[e], h0, h1);
        // u - hi is exact in fp32
        lp[e] = pack2(fma_bf16(h0, kBf16MinusOne, acc[2 * e]),
                      fma_bf16(h1, kBf16MinusOne, acc[2 * e + 1]));
      }
      const uint32_t off = swz_offset(r, j * 16, kRowBytes);
      *reinterpret_cast<uint4*>(smem + L.off_u + off) = hi4;
      *reinterpret_cast<uint4*>(smem + L.off_u + L.u_bytes + off) = lo4;
    }
  };
  auto conv = [&](int hh) {
    if (part == 0)
      conv_part(hh, std::integral_constant<int, 0>{});
    else
      conv_part(hh, std::integral_constant<int, 1>{});
  };

  auto issue_mma = [&](int hh) {
    const uint32_t dt = tmem + (hh & 1) * D;
    const uint32_t wb = w_base + hh * L.w_bytes;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_ss(dt, make_smem_desc(u_hi + kk * 32, 16, kSbo, kSwz),
             make_smem_desc(wb + kk * 32, 16, kSbo, kSwz), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      mma_ss(dt, make_smem_desc(u_lo + kk * 32, 16, kSbo, kSwz),
             make_smem_desc(wb + kk * 32, 16, kSbo, kSwz), idesc, 1u);
    mma_commit(&mma_done[hh & 1]);
  };

  auto epilogue = [&](int hh) {
    const uint32_t col = (hh & 1) * D + part * Q4;
    uint32_t ya[Q4], yb[Q4];                 // channels part*Q4 + e and D/2 + part*Q4 + e
    if constexpr (Q4 == 8) {
      tmem_ld8(trow + col, ya);
      tmem_ld8(trow + col + D / 2, yb);
    } else {
      tmem_ld16(trow + col, ya);
      tmem_ld16(trow + col + D / 2, yb);
    }
    tmem_wait_ld();
    if (t >= S) return;
    const int i0 = part * Q4;
    float lo[Q4], hi[Q4];
#pragma unroll
    for (int e = 0; e < Q4; ++e) {
      lo[e] = __uint_as_float(ya[e]);
      hi[e] = __uint_as_float(yb[e]);
    }
    if (a.qk_mean == 2) {
      // "self" reading: y = (y + own pre-conv value) / 2 over channels c0 + e
      // (slot hh holds this head's q~, or k~ for the key head)
      auto self_mean = [&](float (&y)[Q4], int c0) {
#pragma unroll
        for (int q8 = 0; q8 < Q4 / 8; ++q8) {
          const uint4 ow = *zchunk(hh, r + kPtHalo, c0 / 8 + q8);
          const uint32_t* op = reinterpret_cast<const uint32_t*>(&ow);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            uint16_t o0, o1;
            halves(op[e], o0, o1);
            y[q8 * 8 + 2 * e] = fma_bf16(o0, kBf16Half, 0.5f * y[q8 * 8 + 2 * e]);
            y[q8 * 8 + 2 * e + 1] = fma_bf16(o1, kBf16Half, 0.5f * y[q8 * 8 + 2 * e + 1]);
          }
        }
      };
      self_mean(lo, i0);
      self_mean(hi, i0 + D / 2);
    } else if (a.qk_mean) {
      const bool is_q = hh < G;
      // y[e] += (q~ + k~) / 2 over channels c0 + e (q~: this head, or the
      // mean of the group's query heads for the key head), as fp32 FMAs on the
      // staged bf16 values
      auto add_mean = [&](float (&y)[Q4], int c0) {
#pragma unroll
        for (int q8 = 0; q8 < Q4 / 8; ++q8) {
          const uint4 kw = *zchunk(G, r + kPtHalo, c0 / 8 + q8);
          const uint32_t* kp = reinterpret_cast<const uint32_t*>(&kw);
          if (is_q) {
            const uint4 qw = *zchunk(hh, r + kPtHalo, c0 / 8 + q8);
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(&qw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint16_t q0, q1, k0, k1;
              halves(qp[e], q0, q1);
              halves(kp[e], k0, k1);
              y[q8 * 8 + 2 * e] = fma_bf16(k0, kBf16Half, fma_bf16(q0, kBf16Half, y[q8 * 8 + 2 * e]));
              y[q8 * 8 + 2 * e + 1] =
                  fma_bf16(k1, kBf16Half, fma_bf16(q1, kBf16Half, y[q8 * 8 + 2 * e + 1]));
            }
          } else {
            float sq[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) sq[e] = 0.f;
            for (int hl = 0; hl < G; ++hl) {
              const uint4 qw = *zchunk(hl, r + kPtHalo, c0 / 8 + q8);
              const uint32_t* qp = reinterpret_cast<const uint32_t*>(&qw);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint16_t q0, q1;
                halves(qp[e], q0, q1);
                sq[2 * e] = add_bf16(q0, sq[2 * e]);
                sq[2 * e + 1] = add_bf16(q1, sq[2 * e + 1]);
              }
            }
            const float hg = 0.5f / static_cast<float>(G);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              uint16_t k0, k1;
              halves(kp[e], k0, k1);
              y[q8 * 8 + 2 * e] = fma_bf16(k0, kBf16Half, fmaf(sq[2 * e], hg, y[q8 * 8 + 2 * e]));
              y[q8 * 8 + 2 * e + 1] =
                  fma_bf16(k1, kBf16Half, fmaf(sq[2 * e + 1], hg, y[q8 * 8 + 2 * e + 1]));
            }
          }
        }
      };
      add_mean(lo, i0);
      add_mean(hi, i0 + D / 2);
    }
    if (a.rope_on) {
#pragma unroll
      for (int e = 0; e < Q4; ++e) {
        const float x0 = lo[e], x1 = hi[e];
        lo[e] = x0 * rc[e] - x1 * rs[e];
        hi[e] = x0 * rs[e] + x1 * rc[e];
      }
    }
    bf16* dst = hh < G ? a.q_out + ((static_cast<int64_t>(b) * S + t) * a.Hq + g * G + hh) * D
                       : a.k_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + t) * D;
#pragma unroll
    for (int q8 = 0; q8 < Q4 / 8; ++q8) {
      uint4 pl, ph;
      pl.x = pack2(lo[q8 * 8 + 0], lo[q8 * 8 + 1]);
      pl.y = pack2(lo[q8 * 8 + 2], lo[q8 * 8 + 3]);
      pl.z = pack2(lo[q8 * 8 + 4], lo[q8 * 8 + 5]);
      pl.w = pack2(lo[q8 * 8 + 6], lo[q8 * 8 + 7]);
      ph.x = pack2(hi[q8 * 8 + 0], hi[q8 * 8 + 1]);
      ph.y = pack2(hi[q8 * 8 + 2], hi[q8 * 8 + 3]);
      ph.z = pack2(hi[q8 * 8 + 4], hi[q8 * 8 + 5]);
      ph.w = pack2(hi[q8 * 8 + 6], hi[q8 * 8 + 7]);
      *reinterpret_cast<uint4*>(dst + i0 + q8 * 8) = pl;
      *reinterpret_cast<uint4*>(dst + D / 2 + i0 + q8 * 8) = ph;
    }
  };

  for (int hh = 0; hh < NH; ++hh) {
    if (hh > 0) {
      // MMA(hh - 1) complete: U may be overwritten, accumulator (hh - 1) & 1 is final
      ok = ok && mbar_wait(&mma_done[(hh - 1) & 1], ((hh - 1) >> 1) & 1, &abort_flag, a.dev_err);
      tc_fence_after();
    }
    // query head hh's rows (head 0's and the key head's came with the first barrier)
    if (hh > 0 && hh < G) ok = ok && mbar_wait(&ld_bar[hh], 0, &abort_flag, a.dev_err);
    if (ok) conv(hh);
    fence_proxy_async_smem();   // U is read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ok = ok && !abort_flag;
    if (ok && tid == 0) issue_mma(hh);
    if (ok && hh > 0) epilogue(hh - 1);
  }
  ok = ok && mbar_wait(&mma_done[(NH - 1) & 1], ((NH - 1) >> 1) & 1, &abort_flag, a.dev_err);
  tc_fence_after();
  if (ok) epilogue(NH - 1);
  // 3. value-shift rows loaded at the start
#pragma unroll
  for (int q = 0; q < kVPer; ++q) {
    const int idx = tid + q * kPtThreads;
    const int tl = idx / NCH, i = (idx % NCH) * 8;
    const int tv = t0 + tl;
    if (tv < S)
      *reinterpret_cast<uint4*>(a.v_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + tv) * D +
                                i) = vreg[q];
  }

  // 4. decode state, written by the CTA that holds position S-1 (rows S-KH .. S-1
  // are staged; rows before position 0 are zero).
  if (a.len != nullptr && t0 <= S - 1 && S - 1 < t0 + kPtTT) {
    const int KH = K - 1, Hq = a.Hq, Hkv = a.Hkv;
    for (int rr = 0; rr < KH; ++rr) {
      const int srow = S - KH + rr - t0 + kPtHalo;
      for (int c = tid; c < QC + D; c += kPtThreads) {
        const int h = c / D, ch = c % D;   // slot G: the key head
        const bf16 v = reinterpret_cast<const bf16*>(zchunk(h, srow, ch / 8))[ch % 8];
        if (c < QC)
          a.hist_q[(static_cast<int64_t>(b) * KH + rr) * Hq * D + qcol0 + c] = v;
        else
          a.hist_k[(static_cast<int64_t>(b) * KH + rr) * Hkv * D + g * D + (c - QC)] = v;
      }
    }
    if (a.v_prev)
      for (int i = tid; i < D; i += kPtThreads)
        a.v_prev[static_cast<int64_t>(b) * Hkv * D + g * D + i] =
            src_b[static_cast<int64_t>(S - 1) * ld + vcol0 + i];
    if (g == 0 && tid == 0) a.len[b] = S;
  }

  if (abort_flag && tid == 0) {
    // Do not release TMEM while an MMA might still write it, nor leave while
    // copies into this CTA's shared memory are in flight (bounded waits).
    mma_commit(drain);
    const long long c0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - c0 < kWaitLimitCycles) {
    }
    for (int h = 0; h < G; ++h) {
      const long long c1 = clock64();
      while (!mbar_try_wait(&ld_bar[h], 0) && clock64() - c1 < kWaitLimitCycles) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * D);
  }
}

template <int D>
cudaError_t launch_d(const PreAttnArgs<bf16>& a, cudaStream_t stream) {
  const PtLayout L = pt_layout(D, a.G);
  const CUtensorMapSwizzle swz = (D == 32) ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tmZ, tmWq, tmWk;
  {
    // q~ | k~ | v~ as [B][S][src_ld]: boxes of 131 rows x D columns
    const uint64_t dims[3] = {static_cast<uint64_t>(a.src_ld), static_cast<uint64_t>(a.S),
                              static_cast<uint64_t>(a.B)};
    const uint64_t st[2] = {static_cast<uint64_t>(a.src_ld) * 2,
                            static_cast<uint64_t>(a.S) * a.src_ld * 2};
    const uint32_t box[3] = {static_cast<uint32_t>(D), kPtTT + kPtHalo, 1};
    if (!encode_tensor_map(&tmZ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, a.src, dims, st, box, swz))
      return cudaErrorInvalidValue;
  }
  {
    // channel-mix weights [heads * D][D]: one D x D tile per head
    const uint64_t dq[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.Hq) * D};
    const uint64_t dk[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.Hkv) * D};
    const uint64_t st[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(D), static_cast<uint32_t>(D)};
    if (!encode_tensor_map(&tmWq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.wq_chan, dq, st, box, swz) ||
        !encode_tensor_map(&tmWk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.wk_chan, dk, st, box, swz))
      return cudaErrorInvalidValue;
  }
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(pre_attn_tc_kernel<D>),
                                       static_cast<int>(L.bytes));
  if (e != cudaSuccess) return e;
  dim3 grid((a.S + kPtTT - 1) / kPtTT, a.Hkv, a.B);
  const cudaError_t el = launch_pdl(pre_attn_tc_kernel<D>, grid, dim3(kPtThreads), L.bytes,
                                    stream, tmZ, tmWq, tmWk, a);
  count_launches(1);
  return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace

bool pre_attn_tc_supported(const PreAttnArgs<bf16>& a) {
  if (a.d != 32 && a.d != 64) return false;
  if (a.channel_conv) return false;   // per-tap matrices: the CUDA-core kernel
  if (a.K < 1 || a.K > 4 || a.wq_chan == nullptr || a.wk_chan == nullptr) return false;
  if (a.wq_seq == nullptr || a.wk_seq == nullptr) return false;
  // TMA and bulk copies: 16-byte aligned bases and row pitches
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(a.src) || !al16(a.wq_chan) || !al16(a.wk_chan) || !al16(a.wq_seq) || !al16(a.wk_seq))
    return false;
  if ((a.src_ld * 2) % 16 != 0 || a.S > (1 << 30)) return false;
  return pt_layout(a.d, a.G).bytes <= 227 * 1024;
}

cudaError_t launch_pre_attn_tc(const PreAttnArgs<bf16>& a, cudaStream_t stream) {
  return a.d == 32 ? launch_d<32>(a, stream) : launch_d<64>(a, stream);
}

}  // namespace ccgqa
