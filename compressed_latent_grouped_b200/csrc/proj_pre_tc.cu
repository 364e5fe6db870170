// Latent projection fused with the pre-attention steps (bf16, heads of dim
// 32): x -> q~ | k~ | v~ on the 5th-generation tensor core, then, without a
// trip through HBM, the causal sequence conv, the per-head channel mix, QK-mean,
// RoPE and value-shift ("Compressed Convolutional Attention", Methodologie
// items 1-4; the page's own kernel fuses the conv with the attention that
// follows it).
//
// One CTA owns one kv group of one sequence over 128 projection rows: the 125
// positions [t0, t0 + 125) it writes and the 3 rows before them that the conv
// reaches back to (recomputed by the neighbouring CTA's MMA as well; rows
// before position 0 or past S come back from the TMA unit as zeros, which is
// the conv's zero padding).
//   1. GEMM: warp 0 streams 64-column blocks of x (128 rows) and of the
//      group's (G + 2) d rows of W_qkv (its G query heads, key head and value
//      head: three TMA boxes) through a ring of shared-memory stages; one
//      thread of warp 1 issues tcgen05.mma (M = 128, N = (G + 2) d, K = 16)
//      into TMEM.  Meanwhile the other threads load the mix weights and taps
//      and form their rotary cos / sin.
//   2. The accumulator is read back, rounded to bf16 as the stand-alone GEMM
//      rounds its output, and written into per-head row tiles in shared memory
//      (over the ring, which the GEMM no longer needs).
//   3. Per head, as the stand-alone tensor-core pre-attention kernel: conv on
//      the CUDA cores from the staged rows, split u = hi + lo, mix
//      Y = U_hi W^T + U_lo W^T on the tensor core (into the TMEM columns the
//      GEMM accumulator used), then QK-mean, RoPE and the bf16 store; the
//      epilogue of head h - 1 runs while the MMA of head h does.
//   4. value-shift rows and, in the CTA holding position S - 1, the decode
//      state, all from the staged rows.
// Every wait is bounded; no cluster multicast is used.
#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace ccgqa {
namespace {

using namespace sm100;

constexpr int kPpThreads = 256;
constexpr int kPpM = 128;      // projection rows per CTA == MMA M == TMEM lanes
constexpr int kPpHalo = 3;     // the conv reaches back K - 1 <= 3 rows
constexpr int kPpOut = kPpM - kPpHalo;   // positions written per CTA
constexpr int kPpBK = 64;      // GEMM K block (one 128-byte swizzle row of bf16)
constexpr int kPpD = 32;       // head dim this kernel takes
constexpr uint32_t kPpRow = kPpD * 2;    // bytes of a staged head row (64B swizzle)

struct PpLayout {
  uint32_t nz;                 // GEMM N: (G + 2) d
  uint32_t a_bytes, b_bytes, stage_bytes;
  uint32_t zh_bytes, u_bytes, w_bytes;
  uint32_t off_z, off_u;       // phase 2 / 3, over the ring
  uint32_t off_w, off_tr, off_ws, off_bar, bytes;
};

// Byte layout of the dynamic shared memory (from a 1024-byte aligned base).
// The ring [0, stages x stage) is reused once the GEMM is done: the staged head
// rows (slots 0..G-1 the query heads, G the key head, G+1 the value head; 128
// rows of 64 bytes each) and the U_hi / U_lo tiles of the mix.
__host__ __device__ inline PpLayout pp_layout(int G, int stages) {
  PpLayout L;
  L.nz = static_cast<uint32_t>(G + 2) * kPpD;
  L.a_bytes = kPpM * kPpBK * 2;
  L.b_bytes = L.nz * kPpBK * 2;
  L.stage_bytes = (L.a_bytes + L.b_bytes + 1023u) & ~1023u;
  L.zh_bytes = kPpM * kPpRow;
  L.u_bytes = kPpM * kPpRow;
  L.w_bytes = kPpD * kPpRow;
  L.off_z = 0;
  L.off_u = L.off_z + static_cast<uint32_t>(G + 2) * L.zh_bytes;
  const uint32_t ring = static_cast<uint32_t>(stages) * L.stage_bytes;
  const uint32_t over = L.off_u + 2 * L.u_bytes;
  L.off_w = ring > over ? ring : over;                           // mix weights W_h, h = 0..G
  L.off_tr = L.off_w + static_cast<uint32_t>(G + 1) * L.w_bytes;  // raw taps
  L.off_ws = (L.off_tr + static_cast<uint32_t>(G + 1) * kPpD * 4 * 2 + 15u) & ~15u;
  L.off_bar = L.off_ws + static_cast<uint32_t>(G + 1) * kPpD * 8;  // [(G+1) d][4] bf16 taps
  L.bytes = L.off_bar + 8 * (2 * stages + 6) + 16 + 1024;         // barriers, TMEM slot, slack
  return L;
}

// d = a * b + c for bf16 a, b and fp32 c, d (the product of two bf16 values is
// exact in fp32, so this equals fmaf(float(a), float(b), c)).
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

// ------------------------------------------------------------------ per-head work
// Shared by both forms.  Staged head rows: slot h (0..G-1 the query heads, G
// the key head, G+1 the value head) holds 128 rows of 64 bytes at z + h zh,
// row rr = position t0 - 3 + rr, 64B-swizzled.

// 16 bytes at channel chunk c of slot h, staged row rr
__device__ __forceinline__ const uint4* pp_zchunk(const uint8_t* z, uint32_t zh, int h, int rr,
                                                  int c) {
  return reinterpret_cast<const uint4*>(z + h * zh + swz_offset(rr, c * 16, kPpRow));
}

// conv of head hh for chunks j = P, P + 2, ... of output row r: u = sum_k w[c, k]
// z[t - k, c] by fp32 FMAs on the bf16 operands (taps in order k = 0..3), then
// u = hi + lo in bf16 into the U_hi / U_lo A tiles; rows past the CTA's output
// get zeros
template <int P>
__device__ __forceinline__ void pp_conv(const uint8_t* z, uint32_t zh, const uint2* ws,
                                        uint8_t* u_hi, uint32_t u_bytes, int hh, int r,
                                        bool row_out) {
  constexpr int D = kPpD, NCH = D / 8;
#pragma unroll
  for (int j = P; j < NCH; j += 2) {
    uint4 hi4 = make_uint4(0, 0, 0, 0), lo4 = make_uint4(0, 0, 0, 0);
    if (row_out) {
      const uint4* tw = reinterpret_cast<const uint4*>(ws + hh * D + j * 8);   // 2 channels each
      uint4 t4[4], zz[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) t4[q] = tw[q];
#pragma unroll
      for (int k = 0; k < 4; ++k) zz[k] = *pp_zchunk(z, zh, hh, r + kPpHalo - k, j);
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
        float s = fma_bf16(zv[0], w[0], 0.f);
#pragma unroll
        for (int k = 1; k < 4; ++k) s = fma_bf16(zv[k], w[k], s);
        acc[e] = s;
      }
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
    }
    const uint32_t off = swz_offset(r, j * 16, kPpRow);
    *reinterpret_cast<uint4*>(u_hi + off) = hi4;
    *reinterpret_cast<uint4*>(u_hi + u_bytes + off) = lo4;
  }
}

// epilogue of head hh for output row r (position t): the mixed channels
// part*Q4 + e and d/2 + part*Q4 + e from TMEM at column tcol (warp-collective
// loads), QK-mean from the staged pre-conv rows, RoPE with this thread's
// (cos, sin), bf16 store into q (query heads) or the cache's k rows
__device__ __forceinline__ void pp_epilogue(const uint8_t* z, uint32_t zh, uint32_t tcol, int hh,
                                            int r, int part, int t, bool row_out,
                                            const float (&rc)[kPpD / 4],
                                            const float (&rs)[kPpD / 4],
                                            const PreAttnArgs<bf16>& a, int b, int g) {
  constexpr int D = kPpD, Q4 = D / 4;
  const int G = a.G;
  uint32_t ya[Q4], yb[Q4];
  tmem_ld8(tcol, ya);
  tmem_ld8(tcol + D / 2, yb);
  tmem_wait_ld();
  if (t >= a.S || !row_out) return;
  const int i0 = part * Q4;
  float lo[Q4], hi[Q4];
#pragma unroll
  for (int e = 0; e < Q4; ++e) {
    lo[e] = __uint_as_float(ya[e]);
    hi[e] = __uint_as_float(yb[e]);
  }
  const int rr = r + kPpHalo;                // this position's staged row
  if (a.qk_mean == 2) {
    // "self" reading: y = (y + own pre-conv value) / 2 over channels c0 + e
    auto self_mean = [&](float (&y)[Q4], int c0) {
      const uint4 ow = *pp_zchunk(z, zh, hh, rr, c0 / 8);
      const uint32_t* op = reinterpret_cast<const uint32_t*>(&ow);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint16_t o0, o1;
        halves(op[e], o0, o1);
        y[2 * e] = fma_bf16(o0, kBf16Half, 0.5f * y[2 * e]);
        y[2 * e + 1] = fma_bf16(o1, kBf16Half, 0.5f * y[2 * e + 1]);
      }
    };
    self_mean(lo, i0);
    self_mean(hi, i0 + D / 2);
  } else if (a.qk_mean) {
    const bool is_q = hh < G;
    // y[e] += (q~ + k~) / 2 over channels c0 + e (q~: this head, or the mean of
    // the group's query heads for the key head), as fp32 FMAs on the bf16 rows
    auto add_mean = [&](float (&y)[Q4], int c0) {
      const uint4 kw = *pp_zchunk(z, zh, G, rr, c0 / 8);
      const uint32_t* kp = reinterpret_cast<const uint32_t*>(&kw);
      if (is_q) {
        const uint4 qw = *pp_zchunk(z, zh, hh, rr, c0 / 8);
        const uint32_t* qp = reinterpret_cast<const uint32_t*>(&qw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint16_t q0, q1, k0, k1;
          halves(qp[e], q0, q1);
          halves(kp[e], k0, k1);
          y[2 * e] = fma_bf16(k0, kBf16Half, fma_bf16(q0, kBf16Half, y[2 * e]));
          y[2 * e + 1] = fma_bf16(k1, kBf16Half, fma_bf16(q1, kBf16Half, y[2 * e + 1]));
        }
      } else {
        float sq[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) sq[e] = 0.f;
        for (int hl = 0; hl < G; ++hl) {
          const uint4 qw = *pp_zchunk(z, zh, hl, rr, c0 / 8);
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
          y[2 * e] = fma_bf16(k0, kBf16Half, fmaf(sq[2 * e], hg, y[2 * e]));
          y[2 * e + 1] = fma_bf16(k1, kBf16Half, fmaf(sq[2 * e + 1], hg, y[2 * e + 1]));
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
  bf16* dst = hh < G ? a.q_out + ((static_cast<int64_t>(b) * a.S + t) * a.Hq + g * G + hh) * D
                     : a.k_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + t) * D;
  uint4 pl, ph;
  pl.x = pack2(lo[0], lo[1]);
  pl.y = pack2(lo[2], lo[3]);
  pl.z = pack2(lo[4], lo[5]);
  pl.w = pack2(lo[6], lo[7]);
  ph.x = pack2(hi[0], hi[1]);
  ph.y = pack2(hi[2], hi[3]);
  ph.z = pack2(hi[4], hi[5]);
  ph.w = pack2(hi[6], hi[7]);
  *reinterpret_cast<uint4*>(dst + i0) = pl;
  *reinterpret_cast<uint4*>(dst + D / 2 + i0) = ph;
}

// value-shift rows of positions [t0, t0 + 125): v[t, :d/2] = v~[t, :d/2],
// v[t, d/2:] = v~[t-1, d/2:] (whole-head reading: every channel from t - 1 when
// the group's kv head is one of the last floor(Hkv / 2)); v~ of position -1 is
// the zero row the TMA unit filled in.  Work items first, first + step, ...
__device__ __forceinline__ void pp_value_shift(const uint8_t* z, uint32_t zh,
                                               const PreAttnArgs<bf16>& a, int b, int g, int t0,
                                               int first, int step) {
  constexpr int D = kPpD, NCH = D / 8;
  const bool shift_head = a.value_shift == 2 && g >= a.Hkv - a.Hkv / 2;
  for (int idx = first; idx < kPpOut * NCH; idx += step) {
    const int tl = idx / NCH, c = idx % NCH;
    const int tv = t0 + tl;
    if (tv >= a.S) continue;
    const bool prev = (a.value_shift == 1 && c * 8 >= D / 2) || shift_head;
    const uint4 v = *pp_zchunk(z, zh, a.G + 1, tl + kPpHalo - (prev ? 1 : 0), c);
    *reinterpret_cast<uint4*>(a.v_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + tv) * D +
                              c * 8) = v;
  }
}

// decode state, written by the tile that holds position S - 1: the last K - 1
// pre-conv q~ / k~ rows (staged rows; rows before position 0 are zero), v~ of
// position S - 1 and len
__device__ __forceinline__ void pp_decode_state(const uint8_t* z, uint32_t zh,
                                                const PreAttnArgs<bf16>& a, int b, int g, int t0,
                                                int first, int step) {
  constexpr int D = kPpD;
  const int S = a.S, G = a.G, QC = G * D;
  if (a.len == nullptr || t0 > S - 1 || S - 1 >= t0 + kPpOut) return;
  const int KH = a.K - 1, Hq = a.Hq, Hkv = a.Hkv, qcol0 = g * QC;
  for (int rr = 0; rr < KH; ++rr) {
    const int srow = S - KH + rr - t0 + kPpHalo;
    for (int c = first; c < QC + D; c += step) {
      const int h = c / D, ch = c % D;   // slot G: the key head
      const bf16 v = reinterpret_cast<const bf16*>(pp_zchunk(z, zh, h, srow, ch / 8))[ch % 8];
      if (c < QC)
        a.hist_q[(static_cast<int64_t>(b) * KH + rr) * Hq * D + qcol0 + c] = v;
      else
        a.hist_k[(static_cast<int64_t>(b) * KH + rr) * Hkv * D + g * D + (c - QC)] = v;
    }
  }
  if (a.v_prev)
    for (int i = first; i < D; i += step)
      a.v_prev[static_cast<int64_t>(b) * Hkv * D + g * D + i] =
          reinterpret_cast<const bf16*>(pp_zchunk(z, zh, G + 1, S - 1 - t0 + kPpHalo, i / 8))[i % 8];
  if (g == 0 && first == 0) a.len[b] = S;
}

// ------------------------------------------------------------------ persistent
// The persistent, warp-specialised form (G <= 4, where its buffers fit in shared
// memory): one CTA per SM walks tiles
// c, c + grid, ...; warp 0 streams the GEMM operands through a ring that runs
// on across tiles, warp 1 accumulates tile i into one of two TMEM accumulators
// (2 (G + 2) d columns, then the two mix accumulators), and warps 2-9 (256
// threads) do the heads of tile i - 1 meanwhile, so the pre-attention work
// hides behind the next tile's GEMM.
constexpr int kPwStages = 3;
constexpr int kPwThreads = 64 + 256;

struct PwLayout {
  uint32_t nz, a_bytes, b_bytes, stage_bytes, zh_bytes, u_bytes, w_bytes;
  uint32_t wset_bytes, rt_bytes;   // one buffer of mix weights, of raw taps
  uint32_t off_z, off_u, off_w, off_rt, off_ws, off_bar, bytes;
};

// ring | staged head rows (G + 2 slots of 128 x 64 B) | U_hi, U_lo | two
// buffers of mix weights (G + 1 tiles of 32 x 64 B each; the next tile's are
// copied in while this tile's are in use) | two buffers of raw taps
// [(G + 1) d][K] | packed taps [(G + 1) d][4] bf16 | barriers
__host__ __device__ inline PwLayout pw_layout(int G) {
  PwLayout L;
  L.nz = static_cast<uint32_t>(G + 2) * kPpD;
  L.a_bytes = kPpM * kPpBK * 2;
  L.b_bytes = L.nz * kPpBK * 2;
  L.stage_bytes = (L.a_bytes + L.b_bytes + 1023u) & ~1023u;
  L.zh_bytes = kPpM * kPpRow;
  L.u_bytes = kPpM * kPpRow;
  L.w_bytes = kPpD * kPpRow;
  L.wset_bytes = static_cast<uint32_t>(G + 1) * L.w_bytes;
  L.rt_bytes = static_cast<uint32_t>(G + 1) * kPpD * 4 * 2;   // room for K = 4
  L.off_z = kPwStages * L.stage_bytes;
  L.off_u = L.off_z + static_cast<uint32_t>(G + 2) * L.zh_bytes;
  L.off_w = L.off_u + 2 * L.u_bytes;
  L.off_rt = L.off_w + 2 * L.wset_bytes;
  L.off_ws = L.off_rt + 2 * L.rt_bytes;
  L.off_bar = L.off_ws + static_cast<uint32_t>(G + 1) * kPpD * 8;
  L.bytes = L.off_bar + 8 * (2 * kPwStages + 8) + 16 + 1024;   // barriers, TMEM slot, slack
  return L;
}

__global__ void __launch_bounds__(kPwThreads, 1)
    proj_pre_ws_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWq,
                       const __grid_constant__ CUtensorMap tmWkv, int E, int n_rb,
                       const __grid_constant__ PreAttnArgs<bf16> a) {
  pdl_enter();
  constexpr int D = kPpD;
  constexpr uint32_t kRowBytes = kPpRow;                // 64-byte rows, 64B swizzle
  constexpr uint32_t kSwz = kSwizzle64B;
  constexpr uint32_t kSbo = 8 * kRowBytes;
  constexpr int NCH = D / 8;                            // 16-byte chunks per row
  constexpr int Q4 = D / 4;                             // rotary pairs per epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = a.G, K = a.K;
  const PwLayout L = pw_layout(G);
  const int NH = G + 1, QC = G * D, NZ = static_cast<int>(L.nz);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_tiles = n_rb * a.Hkv * a.B;
  uint8_t* z = smem + L.off_z;                           // slot h: z + h zh_bytes
  uint2* ws = reinterpret_cast<uint2*>(smem + L.off_ws);   // taps of a channel: 4 bf16
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);   // [kPwStages]
  uint64_t* empty = full + kPwStages;                                // [kPwStages]
  uint64_t* acc_full = empty + kPwStages;                            // [2]
  uint64_t* acc_empty = acc_full + 2;                                // [2], 256 arrivals
  uint64_t* mma_done = acc_empty + 2;                                // [2] mix MMAs
  uint64_t* drain = mma_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag, n_issued;
  const int nkb = (E + kPpBK - 1) / kPpBK;
  // tile t: sequence b, row block rb (positions [125 rb, 125 rb + 125)), kv group g
  auto tile_of = [&](int t, int& b, int& rb, int& g) {
    g = t % a.Hkv;
    rb = (t / a.Hkv) % n_rb;
    b = t / (a.Hkv * n_rb);
  };

  if (tid == 0) {
    for (int s = 0; s < kPwStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 256);
      mbar_init(&mma_done[i], 1);
    }
    mbar_init(drain, 2);   // one commit from each MMA issuer (GEMM, mix)
    abort_flag = 0;
    n_issued = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);   // accumulators at 0 and NZ, the mix accumulators at 2 NZ
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t col_mix = 2 * static_cast<uint32_t>(NZ);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmX);
      prefetch_tensormap(&tmWq);
      prefetch_tensormap(&tmWkv);
      int kg = 0;   // k-blocks issued so far (the ring runs on across tiles)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x) {
        int b, rb, g;
        tile_of(t, b, rb, g);
        const int rq = g * QC, rk = a.Hq * D + g * D, rv = (a.Hq + a.Hkv) * D + g * D;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = kg % kPwStages;
          if (!mbar_wait(&empty[s], ((kg / kPwStages) & 1) ^ 1, &abort_flag, a.dev_err)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], L.a_bytes + L.b_bytes);
          uint8_t* sa = smem + s * L.stage_bytes;
          uint8_t* sb = sa + L.a_bytes;
          tma_load_3d(sa, &tmX, &full[s], kb * kPpBK, rb * kPpOut - kPpHalo, b);
          tma_load_2d(sb, &tmWq, &full[s], kb * kPpBK, rq);
          tma_load_2d(sb + QC * 128, &tmWkv, &full[s], kb * kPpBK, rk);
          tma_load_2d(sb + (QC + D) * 128, &tmWkv, &full[s], kb * kPpBK, rv);
          n_issued = kg + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ GEMM MMA issuer
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(kPpM, NZ, false);
      int kg = 0, i = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < n_tiles; t += gridDim.x, ++i) {
        const int buf = i & 1;
        // the head workers have read this accumulator's previous tile back
        if (!mbar_wait(&acc_empty[buf], ((i >> 1) & 1) ^ 1, &abort_flag, a.dev_err)) break;
        tc_fence_after();
        const uint32_t acc = tmem + buf * NZ;
        for (int kb = 0; kb < nkb; ++kb, ++kg) {
          const int s = kg % kPwStages;
          if (!mbar_wait(&full[s], (kg / kPwStages) & 1, &abort_flag, a.dev_err)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_addr(smem + s * L.stage_bytes);
          const uint32_t b_base = a_base + L.a_bytes;
#pragma unroll
          for (int k = 0; k < kPpBK / 16; ++k) {
            const uint64_t ad = make_smem_desc(a_base + k * 32, 16, 1024, kSwizzle128B);
            const uint64_t bd = make_smem_desc(b_base + k * 32, 16, 1024, kSwizzle128B);
            mma_ss(acc, ad, bd, idesc, (kb | k) != 0);
          }
          mma_commit(&empty[s]);
        }
        if (ok) mma_commit(&acc_full[buf]);
      }
    }
  } else {
    // ------------------------------------------------------------ head workers
    const int ptid = tid - 64;                 // 0..255
    const int wq = warp & 3;                   // TMEM lane quadrant of this warp
    const int r = wq * 32 + lane;              // row == TMEM lane (position t0 + r)
    const int part = (warp - 2) >> 2;          // conv chunks j = part (mod 2); pairs of half `part`
    const bool row_out = r < kPpOut;
    const uint32_t trow = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t u_hi = smem_addr(smem + L.off_u);
    const uint32_t u_lo = u_hi + L.u_bytes;
    const uint32_t w_base = smem_addr(smem + L.off_w);
    const uint32_t idesc = make_idesc_bf16(kPpM, D, false);
    // mix weights W_h [d_out][d_in] of group g into weight buffer wb (the
    // K-major 64B-swizzled B layout) and the group's raw taps into tap buffer
    // wb, by 16-byte asynchronous copies (all four sources 16-byte aligned)
    auto prefetch_weights = [&](int g, int wb) {
      uint8_t* wdst = smem + L.off_w + wb * L.wset_bytes;
      for (int idx = ptid; idx < NH * D * NCH; idx += 256) {
        const int h = idx / (D * NCH), row = (idx / NCH) % D, c = idx % NCH;
        const bf16* src = h < G ? a.wq_chan + (static_cast<int64_t>(g * G + h) * D + row) * D
                                : a.wk_chan + (static_cast<int64_t>(g) * D + row) * D;
        cp_async16(wdst + h * L.w_bytes + swz_offset(row, c * 16, kRowBytes), src + c * 8);
      }
      uint8_t* tdst = smem + L.off_rt + wb * L.rt_bytes;
      const int qb = G * D * K * 2, kbytes = D * K * 2;   // multiples of 64
      const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(a.wq_seq + static_cast<int64_t>(g) * G * D * K);
      const uint8_t* ksrc = reinterpret_cast<const uint8_t*>(a.wk_seq + static_cast<int64_t>(g) * D * K);
      for (int o = ptid * 16; o < qb + kbytes; o += 256 * 16)
        cp_async16(tdst + o, o < qb ? qsrc + o : ksrc + (o - qb));
      cp_async_commit_group();
    };
    bool ok = true;
    int mix_base = 0;                           // mix MMAs issued by this CTA before this tile
    if (blockIdx.x < n_tiles) {
      prefetch_weights(static_cast<int>(blockIdx.x) % a.Hkv, 0);
      cp_async_wait_all_groups();
      named_barrier_sync(1, 256);
    }
    for (int t = blockIdx.x, i = 0; ok && t < n_tiles; t += gridDim.x, ++i) {
      int b, rb, g;
      tile_of(t, b, rb, g);
      const int t0 = rb * kPpOut, tp = t0 + r;
      const int buf = i & 1;
      // (every worker is done with the previous tile's staged rows, U and taps,
      // and this tile's weights and raw taps have landed: the barrier that ends
      // each tile)  Taps as bf16 [channel][4], zero past K.
      const bf16* rt = reinterpret_cast<const bf16*>(smem + L.off_rt + buf * L.rt_bytes);
      for (int hc = ptid; hc < NH * D; hc += 256) {
        uint16_t w4[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) w4[k] = k < K ? __bfloat16_as_ushort(rt[hc * K + k]) : static_cast<uint16_t>(0);
        ws[hc] = make_uint2(w4[0] | (static_cast<uint32_t>(w4[1]) << 16),
                            w4[2] | (static_cast<uint32_t>(w4[3]) << 16));
      }
      // rotary (cos, sin) of this thread's pairs at position t0 + r (angle
      // reduced modulo one turn exactly in 64-bit fixed point)
      float rc[Q4], rs[Q4];
      {
        const int ip = part * Q4;
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
      // the tile's accumulator -> staged bf16 head rows; then it is free again
      ok = mbar_wait(&acc_full[buf], (i >> 1) & 1, &abort_flag, a.dev_err);
      tc_fence_after();
      {
        const int n_slots = G + 2, half_slots = (n_slots + 1) / 2;
        const int s_lo = part == 0 ? 0 : half_slots, s_hi = part == 0 ? half_slots : n_slots;
        for (int sl = s_lo; sl < s_hi; ++sl) {
          uint32_t v[32];
          tmem_ld32(trow + buf * NZ + sl * D, v);
          tmem_wait_ld();
          if (ok) {
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
              uint4 pk;
              pk.x = pack2(__uint_as_float(v[c * 8 + 0]), __uint_as_float(v[c * 8 + 1]));
              pk.y = pack2(__uint_as_float(v[c * 8 + 2]), __uint_as_float(v[c * 8 + 3]));
              pk.z = pack2(__uint_as_float(v[c * 8 + 4]), __uint_as_float(v[c * 8 + 5]));
              pk.w = pack2(__uint_as_float(v[c * 8 + 6]), __uint_as_float(v[c * 8 + 7]));
              *reinterpret_cast<uint4*>(z + sl * L.zh_bytes + swz_offset(r, c * 16, kRowBytes)) = pk;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      // the next tile's weights into the other buffers (their last reader, the
      // tile before this one, is done), landing while this tile's heads run
      if (t + static_cast<int>(gridDim.x) < n_tiles)
        prefetch_weights((t + static_cast<int>(gridDim.x)) % a.Hkv, buf ^ 1);
      fence_proxy_async_smem();   // W (copied in at the end of the previous tile) is read by the tensor core
      // one answer for all 256 workers (a worker leaving the loop alone would
      // leave the others at a named barrier)
      ok = !named_barrier_or(1, 256, !ok || abort_flag);
      if (!ok) break;

      // per head, as the one-tile kernel; mix MMA m (m = mix_base + head) goes
      // into accumulator m & 1 and completes on mma_done[m & 1]
      auto issue_mma = [&](int hh, int m) {
        const uint32_t dt = tmem + col_mix + (m & 1) * D;
        const uint32_t wb = w_base + buf * L.wset_bytes + hh * L.w_bytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(dt, make_smem_desc(u_hi + kk * 32, 16, kSbo, kSwz),
                 make_smem_desc(wb + kk * 32, 16, kSbo, kSwz), idesc, kk > 0 ? 1u : 0u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(dt, make_smem_desc(u_lo + kk * 32, 16, kSbo, kSwz),
                 make_smem_desc(wb + kk * 32, 16, kSbo, kSwz), idesc, 1u);
        mma_commit(&mma_done[m & 1]);
      };

      auto epilogue = [&](int hh, int m) {
        pp_epilogue(z, L.zh_bytes, trow + col_mix + (m & 1) * D + part * Q4, hh, r, part, tp,
                    row_out, rc, rs, a, b, g);
      };

      for (int hh = 0; hh < NH; ++hh) {
        const int m = mix_base + hh;
        if (hh > 0) {
          // MMA m - 1 complete: U may be overwritten, accumulator (m - 1) & 1 is final
          ok = ok && mbar_wait(&mma_done[(m - 1) & 1], ((m - 1) >> 1) & 1, &abort_flag, a.dev_err);
          tc_fence_after();
        }
        if (ok) {
          if (part == 0)
            pp_conv<0>(z, L.zh_bytes, ws, smem + L.off_u, L.u_bytes, hh, r, row_out);
          else
            pp_conv<1>(z, L.zh_bytes, ws, smem + L.off_u, L.u_bytes, hh, r, row_out);
        }
        fence_proxy_async_smem();   // U is read by the tensor core
        tc_fence_before();
        ok = !named_barrier_or(1, 256, !ok || abort_flag);
        tc_fence_after();
        if (ok && ptid == 0) issue_mma(hh, m);
        __syncwarp();
        if (ok && hh > 0) epilogue(hh - 1, m - 1);
      }
      const int m_last = mix_base + NH - 1;
      ok = ok && mbar_wait(&mma_done[m_last & 1], (m_last >> 1) & 1, &abort_flag, a.dev_err);
      ok = __all_sync(0xffffffffu, ok);   // the epilogue's TMEM loads are warp-collective
      tc_fence_after();
      if (ok) epilogue(NH - 1, m_last);
      mix_base += NH;

      pp_value_shift(z, L.zh_bytes, a, b, g, t0, ptid, 256);
      pp_decode_state(z, L.zh_bytes, a, b, g, t0, ptid, 256);
      // end of the tile: the next tile's weights have landed, the staged rows
      // are free, and one answer for all workers
      cp_async_wait_all_groups();
      ok = !named_barrier_or(1, 256, !ok || abort_flag);
    }
    cp_async_wait_all_groups();   // no copy into shared memory outlives the loop
  }

  if (abort_flag) {
    // Do not release TMEM while an MMA might still write it (the GEMM issuer's
    // and the mix issuer's own MMAs), nor leave while the ring's last loads
    // are in flight (bounded waits).
    if ((warp == 1 && lane == 0) || tid == 64) {
      mma_commit(drain);
      const long long c0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - c0 < kWaitLimitCycles) {
      }
    }
    if (tid == 0) {
      const int n = n_issued;
      for (int kg = n > kPwStages ? n - kPwStages : 0; kg < n; ++kg) {
        const long long c2 = clock64();
        while (!mbar_try_wait(&full[kg % kPwStages], (kg / kPwStages) & 1) &&
               clock64() - c2 < kWaitLimitCycles) {
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// kPpStages = 3 (one CTA per SM) when the grid is at most one wave; 2 (about
// 97 KB of shared memory at G = 4, so two CTAs share an SM and one's GEMM runs
// while the other works on its heads) otherwise.
template <int kPpStages>
__global__ void __launch_bounds__(kPpThreads, kPpStages == 2 ? 2 : 1)
    proj_pre_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmWq,
                       const __grid_constant__ CUtensorMap tmWkv,
                       const __grid_constant__ CUtensorMap tmMq,
                       const __grid_constant__ CUtensorMap tmMk, int E,
                       const __grid_constant__ PreAttnArgs<bf16> a) {
  pdl_enter();
  constexpr int D = kPpD;
  constexpr uint32_t kRowBytes = kPpRow;                // 64-byte rows, 64B swizzle
  constexpr uint32_t kSwz = kSwizzle64B;
  constexpr uint32_t kSbo = 8 * kRowBytes;
  constexpr int NCH = D / 8;                            // 16-byte chunks per row
  constexpr int Q4 = D / 4;                             // rotary pairs per epilogue thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int G = a.G, K = a.K;
  const PpLayout L = pp_layout(G, kPpStages);
  const int NH = G + 1, QC = G * D, NZ = static_cast<int>(L.nz);
  const int b = blockIdx.z, g = blockIdx.y, t0 = blockIdx.x * kPpOut;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* z = smem + L.off_z;                           // slot h: z + h zh_bytes
  uint2* ws = reinterpret_cast<uint2*>(smem + L.off_ws);   // taps of a channel: 4 bf16
  const bf16* tr = reinterpret_cast<const bf16*>(smem + L.off_tr);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.off_bar);   // [kPpStages]
  uint64_t* empty = full + kPpStages;                                // [kPpStages]
  uint64_t* acc_full = empty + kPpStages;
  uint64_t* wl_bar = acc_full + 1;                                   // mix weights and taps
  uint64_t* mma_done = wl_bar + 1;                                   // [2]
  uint64_t* drain = mma_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ int abort_flag, n_issued;   // n_issued: k-blocks whose loads the producer issued

  const int nkb = (E + kPpBK - 1) / kPpBK;

  if (tid == 0) {
    for (int s = 0; s < kPpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(wl_bar, 1);
    mbar_init(&mma_done[0], 1);
    mbar_init(&mma_done[1], 1);
    mbar_init(drain, 2);   // one commit from each MMA issuer (GEMM: thread 32, mix: thread 0)
    abort_flag = 0;
    n_issued = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 256);   // the GEMM accumulator, later the two mix accumulators
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  // 1. GEMM Z[128, NZ] = x[t0 - 3 .. t0 + 124] W_g^T
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmX);
    prefetch_tensormap(&tmWq);
    prefetch_tensormap(&tmWkv);
    prefetch_tensormap(&tmMq);
    prefetch_tensormap(&tmMk);
    // mix weights (straight into the K-major swizzled B layout) and taps
    const uint32_t tq = static_cast<uint32_t>(G) * D * K * 2, tk = static_cast<uint32_t>(D) * K * 2;
    mbar_arrive_expect_tx(wl_bar, tq + tk + NH * L.w_bytes);
    bulk_load(smem + L.off_tr, a.wq_seq + static_cast<int64_t>(g) * G * D * K, tq, wl_bar);
    bulk_load(smem + L.off_tr + tq, a.wk_seq + static_cast<int64_t>(g) * D * K, tk, wl_bar);
    for (int h = 0; h < G; ++h)
      tma_load_2d(smem + L.off_w + h * L.w_bytes, &tmMq, wl_bar, 0, (g * G + h) * D);
    tma_load_2d(smem + L.off_w + G * L.w_bytes, &tmMk, wl_bar, 0, g * D);
    const int rq = g * QC, rk = a.Hq * D + g * D, rv = (a.Hq + a.Hkv) * D + g * D;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kPpStages;
      if (!mbar_wait(&empty[s], ((kb / kPpStages) & 1) ^ 1, &abort_flag, a.dev_err)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&full[s], L.a_bytes + L.b_bytes);
      uint8_t* sa = smem + s * L.stage_bytes;
      uint8_t* sb = sa + L.a_bytes;
      tma_load_3d(sa, &tmX, &full[s], kb * kPpBK, t0 - kPpHalo, b);
      tma_load_2d(sb, &tmWq, &full[s], kb * kPpBK, rq);
      tma_load_2d(sb + QC * 128, &tmWkv, &full[s], kb * kPpBK, rk);
      tma_load_2d(sb + (QC + D) * 128, &tmWkv, &full[s], kb * kPpBK, rv);
      n_issued = kb + 1;
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(kPpM, NZ, false);
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kPpStages;
      if (!mbar_wait(&full[s], (kb / kPpStages) & 1, &abort_flag, a.dev_err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a_base = smem_addr(smem + s * L.stage_bytes);
      const uint32_t b_base = a_base + L.a_bytes;
#pragma unroll
      for (int k = 0; k < kPpBK / 16; ++k) {
        // K-major, 128B-swizzled: 8-row groups 1024 B apart, a K step of 16
        // bf16 advances 32 B inside the swizzle row
        const uint64_t ad = make_smem_desc(a_base + k * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd = make_smem_desc(b_base + k * 32, 16, 1024, kSwizzle128B);
        mma_ss(tmem, ad, bd, idesc, (kb | k) != 0);
      }
      mma_commit(&empty[s]);
    }
    if (ok) mma_commit(acc_full);
  }
  // RoPE of this thread's epilogue pairs (row tid % 128, pairs of half tid / 128)
  // while the GEMM runs: (cos, sin) of t * theta_i, the angle taken modulo one
  // turn exactly in 64-bit fixed point, then |2 pi f| <= pi.
  float rc[Q4], rs[Q4];
  {
    const int tp = t0 + (tid & (kPpM - 1)), ip = (tid >> 7) * Q4;
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
  // conv taps as bf16 [channel][4], zero past K
  ok = ok && mbar_wait(wl_bar, 0, &abort_flag, a.dev_err);
  for (int hc = tid; hc < NH * D; hc += kPpThreads) {
    uint16_t w4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      w4[k] = k < K ? __bfloat16_as_ushort(tr[hc * K + k]) : static_cast<uint16_t>(0);
    ws[hc] = make_uint2(w4[0] | (static_cast<uint32_t>(w4[1]) << 16),
                        w4[2] | (static_cast<uint32_t>(w4[3]) << 16));
  }
  // 2. accumulator -> staged bf16 head rows (warps w and w + 4 share TMEM lanes
  // 32 (w % 4) .. + 31 and split the slots)
  ok = ok && mbar_wait(acc_full, 0, &abort_flag, a.dev_err);
  __syncwarp();   // lane 0 of warps 0 and 1 ran the GEMM loops: converge before tcgen05.ld
  tc_fence_after();
  {
    const int r = (warp & 3) * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const int n_slots = G + 2, half_slots = (n_slots + 1) / 2;
    const int s_lo = warp < 4 ? 0 : half_slots, s_hi = warp < 4 ? half_slots : n_slots;
    for (int sl = s_lo; sl < s_hi; ++sl) {
      uint32_t v[32];
      tmem_ld32(trow + sl * D, v);
      tmem_wait_ld();
      if (ok) {
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint4 pk;
          pk.x = pack2(__uint_as_float(v[c * 8 + 0]), __uint_as_float(v[c * 8 + 1]));
          pk.y = pack2(__uint_as_float(v[c * 8 + 2]), __uint_as_float(v[c * 8 + 3]));
          pk.z = pack2(__uint_as_float(v[c * 8 + 4]), __uint_as_float(v[c * 8 + 5]));
          pk.w = pack2(__uint_as_float(v[c * 8 + 6]), __uint_as_float(v[c * 8 + 7]));
          *reinterpret_cast<uint4*>(z + sl * L.zh_bytes + swz_offset(r, c * 16, kRowBytes)) = pk;
        }
      }
    }
  }
  // staged rows and taps ready; every read of the accumulator done, so the mix
  // accumulators may take its columns
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  ok = ok && !abort_flag;

  // 3. per head (slots 0..G-1 the query heads, G the key head)
  const int r = tid & (kPpM - 1);          // output row == TMEM lane (position t0 + r)
  const int part = tid >> 7;               // conv chunks j = part (mod 2); pairs of half `part`
  const uint32_t trow = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
  const uint32_t u_hi = smem_addr(smem + L.off_u);
  const uint32_t u_lo = u_hi + L.u_bytes;
  const uint32_t w_base = smem_addr(smem + L.off_w);
  const uint32_t idesc = make_idesc_bf16(kPpM, D, false);
  const int t = t0 + r;
  const bool row_out = r < kPpOut;         // rows 125..127 of the MMA tile are not written
  auto conv = [&](int hh) {
    if (part == 0)
      pp_conv<0>(z, L.zh_bytes, ws, smem + L.off_u, L.u_bytes, hh, r, row_out);
    else
      pp_conv<1>(z, L.zh_bytes, ws, smem + L.off_u, L.u_bytes, hh, r, row_out);
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
    pp_epilogue(z, L.zh_bytes, trow + (hh & 1) * D + part * Q4, hh, r, part, t, row_out, rc, rs,
                a, b, g);
  };

  for (int hh = 0; hh < NH; ++hh) {
    if (hh > 0) {
      // MMA(hh - 1) complete: U may be overwritten, accumulator (hh - 1) & 1 is final
      ok = ok && mbar_wait(&mma_done[(hh - 1) & 1], ((hh - 1) >> 1) & 1, &abort_flag, a.dev_err);
      tc_fence_after();
    }
    if (ok) conv(hh);
    fence_proxy_async_smem();   // U is read by the tensor core
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    ok = __all_sync(0xffffffffu, ok && !abort_flag);   // warp-uniform for the TMEM loads
    if (ok && tid == 0) issue_mma(hh);
    __syncwarp();
    if (ok && hh > 0) epilogue(hh - 1);
  }
  ok = ok && mbar_wait(&mma_done[(NH - 1) & 1], ((NH - 1) >> 1) & 1, &abort_flag, a.dev_err);
  ok = __all_sync(0xffffffffu, ok);   // the epilogue's TMEM loads are warp-collective
  tc_fence_after();
  if (ok) epilogue(NH - 1);

  // 4. value-shift rows; 5. decode state (the CTA holding position S - 1)
  pp_value_shift(z, L.zh_bytes, a, b, g, t0, tid, kPpThreads);
  pp_decode_state(z, L.zh_bytes, a, b, g, t0, tid, kPpThreads);

  if (abort_flag && (tid == 0 || tid == 32)) {
    // Do not release TMEM while an MMA might still write it (each issuer
    // commits its own), nor leave while copies into this CTA's shared memory
    // are in flight (bounded waits).
    mma_commit(drain);
    const long long c0 = clock64();
    while (!mbar_try_wait(drain, 0) && clock64() - c0 < kWaitLimitCycles) {
    }
  }
  if (abort_flag && tid == 0) {
    const long long c1 = clock64();
    while (!mbar_try_wait(wl_bar, 0) && clock64() - c1 < kWaitLimitCycles) {
    }
    // the ring's last loads (earlier ones completed before their stage was reused)
    for (int kb = n_issued > kPpStages ? n_issued - kPpStages : 0; kb < n_issued; ++kb) {
      const long long c2 = clock64();
      while (!mbar_try_wait(&full[kb % kPpStages], (kb / kPpStages) & 1) &&
             clock64() - c2 < kWaitLimitCycles) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

bool proj_pre_tc_supported(const PreAttnArgs<bf16>& a, const bf16* x, const bf16* W, int E) {
  if (a.d != kPpD || a.channel_conv) return false;
  if (a.K < 1 || a.K > 4 || !a.wq_seq || !a.wk_seq || !a.wq_chan || !a.wk_chan) return false;
  if (!x || !W || E <= 0 || E % 8 != 0) return false;   // 16-byte row pitch of x and W
  if (a.G + 2 > 8) return false;                         // GEMM N = (G + 2) d <= 256
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
  if (!al16(x) || !al16(W) || !al16(a.wq_chan) || !al16(a.wk_chan) || !al16(a.wq_seq) ||
      !al16(a.wk_seq))
    return false;
  if (a.S > (1 << 30)) return false;
  return pp_layout(a.G, 3).bytes <= 227 * 1024;
}

cudaError_t launch_proj_pre_tc(const bf16* x, const bf16* W, int E, const PreAttnArgs<bf16>& a,
                               cudaStream_t stream) {
  constexpr int D = kPpD;
  const int N = (a.Hq + 2 * a.Hkv) * D;
  CUtensorMap tmX, tmWq, tmWkv, tmMq, tmMk;
  {
    // x [B][S][E]: boxes of 64 columns x 128 rows of one sequence (rows before
    // position 0 or past S read as zeros)
    const uint64_t dims[3] = {static_cast<uint64_t>(E), static_cast<uint64_t>(a.S),
                              static_cast<uint64_t>(a.B)};
    const uint64_t st[2] = {static_cast<uint64_t>(E) * 2, static_cast<uint64_t>(a.S) * E * 2};
    const uint32_t box[3] = {kPpBK, kPpM, 1};
    if (!encode_tensor_map(&tmX, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, x, dims, st, box,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    // W_qkv [N][E]: the group's query rows in one box, its key and value rows in two
    const uint64_t dims[2] = {static_cast<uint64_t>(E), static_cast<uint64_t>(N)};
    const uint64_t st[1] = {static_cast<uint64_t>(E) * 2};
    const uint32_t bq[2] = {kPpBK, static_cast<uint32_t>(a.G * D)};
    const uint32_t bkv[2] = {kPpBK, static_cast<uint32_t>(D)};
    if (!encode_tensor_map(&tmWq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dims, st, bq,
                           CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tensor_map(&tmWkv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, W, dims, st, bkv,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  }
  {
    // channel-mix weights [heads * D][D]: one D x D tile per head
    const uint64_t dq[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.Hq) * D};
    const uint64_t dk[2] = {static_cast<uint64_t>(D), static_cast<uint64_t>(a.Hkv) * D};
    const uint64_t st[1] = {static_cast<uint64_t>(D) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(D), static_cast<uint32_t>(D)};
    if (!encode_tensor_map(&tmMq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.wq_chan, dq, st, box,
                           CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_tensor_map(&tmMk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.wk_chan, dk, st, box,
                           CU_TENSOR_MAP_SWIZZLE_64B))
      return cudaErrorInvalidValue;
  }
  dim3 grid((a.S + kPpOut - 1) / kPpOut, a.Hkv, a.B);
  const int sms = sm_count();
  if (2 * (a.G + 2) * D + 2 * D <= 512 && pw_layout(a.G).bytes <= 227 * 1024) {
    // persistent: two GEMM accumulators and the two mix accumulators fit in TMEM
    const int n_rb = static_cast<int>(grid.x);
    const int n_tiles = n_rb * a.Hkv * a.B;
    const int pgrid = n_tiles < sms ? n_tiles : sms;
    const PwLayout P = pw_layout(a.G);
    cudaError_t e = allow_smem(reinterpret_cast<const void*>(proj_pre_ws_kernel),
                               static_cast<int>(P.bytes));
    if (e != cudaSuccess) return e;
    const cudaError_t el = launch_pdl(proj_pre_ws_kernel, dim3(pgrid), dim3(kPwThreads), P.bytes,
                                      stream, tmX, tmWq, tmWkv, E, n_rb, a);
    count_launches(1);
    return el != cudaSuccess ? el : cudaGetLastError();
  }
  const bool one_wave = static_cast<int64_t>(grid.x) * grid.y * grid.z <= sms;
  auto kernel = one_wave ? proj_pre_tc_kernel<3> : proj_pre_tc_kernel<2>;
  const PpLayout L = pp_layout(a.G, one_wave ? 3 : 2);
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kernel), static_cast<int>(L.bytes));
  if (e != cudaSuccess) return e;
  const cudaError_t el = launch_pdl(kernel, grid, dim3(kPpThreads), L.bytes, stream, tmX, tmWq,
                                    tmWkv, tmMq, tmMk, E, a);
  count_launches(1);
  return el != cudaSuccess ? el : cudaGetLastError();
}

}  // namespace ccgqa
