// Fused pre-attention kernel: causal sequence conv + per-head channel mix +
// QK-mean + RoPE on q~ and k~, value-shift on v~
// ("Compressed Convolutional Attention", Methodologie items 2-4).
//
// One CTA owns TT consecutive positions of one kv group (its G query heads, its
// key head and its value head) of one sequence, so QK-mean, which mixes the
// group's query heads with its key head, needs no data from other CTAs.
//   1. the group's q~ | k~ | v~ rows [t0 - HALO, t0 + TT) are copied into
//      shared memory with 16-byte cp.async (raw working dtype; the halo rows
//      feed the causal conv and the value-shift);
//   2. per head: the depthwise causal conv, one thread per channel sliding a
//      K-tap register window down its rows, then the channel mix y = W_h u as
//      a register-tiled (4 positions x 4 channels) product, QK-mean from the
//      staged pre-conv rows, RoPE from a per-CTA cos/sin table, one store;
//   3. value-shift: upper half-channels of each value head come from the
//      previous position -- a bit-exact copy out of shared memory;
//   4. the CTA holding the last position writes the decode state.
// All arithmetic in fp32; inputs and outputs in the working dtype.
#include <type_traits>

#include "kernels.h"

namespace ccgqa {
namespace {

constexpr int kPreThreads = 256;

__host__ __device__ inline int round4(int x) { return (x + 3) & ~3; }

struct PreLayout {
  int TT, KH, HALO, R, ZC, US;
  int off_u, off_w, off_cs, off_theta;  // in floats, after the z tile
  size_t z_bytes, bytes;
};

// has_mix: a channel-mix weight is present (else no transposed-weight buffer);
// K == 0: no conv output buffer either.
__host__ __device__ inline PreLayout pre_layout(int TT, int K, int G, int d, int es,
                                                bool has_mix) {
  PreLayout L;
  L.TT = TT;
  L.KH = K > 0 ? K - 1 : 0;
  L.HALO = L.KH > 1 ? L.KH : 1;   // at least one row back for the value-shift
  L.R = TT + L.HALO;
  L.ZC = (G + 2) * d + 16 / es;   // q | k | v channels + one 16-byte pad
  L.US = TT + 4;                  // multiple of 4 for float4 reads
  L.z_bytes = (static_cast<size_t>(L.R) * L.ZC * es + 15) & ~size_t(15);
  L.off_u = 0;
  L.off_w = L.off_u + (K > 0 ? round4(d * L.US) : 0);
  L.off_cs = L.off_w + (K > 0 && has_mix ? round4(d * (d + 2)) : 0);
  L.off_theta = L.off_cs + round4(TT * d);  // cs: TT * d/2 float2
  L.bytes = L.z_bytes + static_cast<size_t>(L.off_theta) * 4 + static_cast<size_t>(d / 2) * 8 + 16;
  return L;
}

template <typename T> struct Vec2;
template <> struct Vec2<float> {
  using type = float2;
  __device__ static type make(float a, float b) { return make_float2(a, b); }
};
template <> struct Vec2<bf16> {
  using type = __nv_bfloat162;
  __device__ static type make(float a, float b) { return __floats2bfloat162_rn(a, b); }
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

template <typename T, int D>
__global__ void __launch_bounds__(kPreThreads)
    pre_attn_kernel(const PreAttnArgs<T> a, const int TT) {
  extern __shared__ float4 smem_f4[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(smem_f4);
  const int b = blockIdx.z, g = blockIdx.y, t0 = blockIdx.x * TT;
  constexpr int d = D, half = D / 2;
  constexpr int WS = D + 2;        // padded row of the transposed channel-mix weight
  const int G = a.G, K = a.K, S = a.S;
  const bool full = a.channel_conv && K > 0;   // per-tap d x d matrices, weights read from L1/L2
  const PreLayout L = pre_layout(TT, K, G, d, sizeof(T),
                                 !full && (a.wq_chan != nullptr || a.wk_chan != nullptr));
  T* z = reinterpret_cast<T*>(smem);                      // [R][ZC]: q | k | v
  float* fs = reinterpret_cast<float*>(smem + L.z_bytes);
  float* u = fs + L.off_u;                                // [d][US]
  float* Wt = fs + L.off_w;                               // [d][d] transposed
  float2* cs = reinterpret_cast<float2*>(fs + L.off_cs);  // [TT][d/2]
  double* theta = reinterpret_cast<double*>(fs + L.off_theta);
  const int HALO = L.HALO, ZC = L.ZC, US = L.US, R = L.R;
  const int tid = threadIdx.x;
  const int64_t ld = a.src_ld;
  const T* src_b = a.src + static_cast<int64_t>(b) * S * ld;
  const int QC = G * d;                   // q channels of the group
  const int qcol0 = g * QC;
  const int kcol0 = a.Hq * d + g * d;
  const int vcol0 = (a.Hq + a.Hkv) * d + g * d;

  // 1. stage rows t0-HALO .. t0+TT-1 of the group's q | k | v channels.
  {
    constexpr int VEC = 16 / sizeof(T);
    const int cq = QC / VEC, ck = d / VEC;            // 16-byte chunks per block
    const int per_row = cq + 2 * ck;
    for (int idx = tid; idx < R * per_row; idx += kPreThreads) {
      const int r = idx / per_row;
      const int c = idx - r * per_row;
      const int t = t0 - HALO + r;
      int col, zc;
      if (c < cq) {
        col = qcol0 + c * VEC;
        zc = c * VEC;
      } else if (c < cq + ck) {
        col = kcol0 + (c - cq) * VEC;
        zc = QC + (c - cq) * VEC;
      } else {
        col = vcol0 + (c - cq - ck) * VEC;
        zc = QC + d + (c - cq - ck) * VEC;
      }
      T* dst = z + r * ZC + zc;
      if (t >= 0 && t < S)
        cp_async16(dst, src_b + static_cast<int64_t>(t) * ld + col);
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  // 2. RoPE table while the copies fly: pair i turns by t * base^(-2i/d).  The
  // angle is formed and reduced modulo one turn in fp64, so long positions
  // keep full precision.
  if (a.rope_on) {
    for (int i = tid; i < half; i += kPreThreads)
      theta[i] = exp2(-(2.0 * i / d) * a.rope_log2_base);
  }
  cp_async_wait_all();
  __syncthreads();
  if (a.rope_on) {
    const double inv_turn = 0.15915494309189533577;  // 1 / (2 pi)
    for (int idx = tid; idx < TT * half; idx += kPreThreads) {
      const int tl = idx / half, i = idx - tl * half;
      double f = static_cast<double>(t0 + tl) * theta[i] * inv_turn;
      f -= rint(f);
      float s, c;
      sincospif(static_cast<float>(2.0 * f), &s, &c);
      cs[idx] = make_float2(c, s);
    }
  }
  __syncthreads();   // the table is read by every head's epilogue

  // 3. per head of the group: G query heads, then the key head.
  constexpr int SEG = 8;                 // rows per conv thread
  const int n_seg = TT / SEG;
  for (int hh = 0; hh <= G; ++hh) {
    const bool is_q = hh < G;
    const int head = is_q ? g * G + hh : g;
    const int cb = hh * d;               // channel offset inside the z tile
    const T* wch_base = is_q ? a.wq_chan : a.wk_chan;
    const T* wch = (K > 0 && wch_base && !full) ? wch_base + static_cast<int64_t>(head) * d * d
                                                : nullptr;
    // the head's per-tap matrices W[head][k] (temporal channel conv)
    const T* wfull = full ? wch_base + static_cast<int64_t>(head) * K * d * d : nullptr;
    // causal depthwise conv: thread = (channel, 8-row segment), taps in registers
    // (no conv: the epilogue reads q~ / k~ straight from the staged rows)
    for (int idx = tid; K > 0 && !full && idx < d * n_seg; idx += kPreThreads) {
      const int j = idx % d, sg = idx / d;
      const int tl0 = sg * SEG;
      const T* zc = z + cb + j;
      if (K > 0) {
        const T* w = (is_q ? a.wq_seq : a.wk_seq) + static_cast<int64_t>(head * d + j) * K;
        float wr[4] = {0.f, 0.f, 0.f, 0.f};
        float win[4] = {0.f, 0.f, 0.f, 0.f};   // win[k] = row tl - k
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (k < K) wr[k] = to_f32(w[k]);
#pragma unroll
        for (int k = 1; k < 4; ++k)
          if (k < K) win[k] = to_f32(zc[(tl0 + HALO - k) * ZC]);
#pragma unroll
        for (int s = 0; s < SEG; ++s) {
          win[0] = to_f32(zc[(tl0 + s + HALO) * ZC]);
          float acc = wr[0] * win[0];
#pragma unroll
          for (int k = 1; k < 4; ++k) acc = fmaf(wr[k], win[k], acc);
          u[j * US + tl0 + s] = acc;
#pragma unroll
          for (int k = 3; k > 0; --k) win[k] = win[k - 1];
        }
      } else {
#pragma unroll
        for (int s = 0; s < SEG; ++s) u[j * US + tl0 + s] = to_f32(zc[(tl0 + s + HALO) * ZC]);
      }
    }
    if (wch) {
      for (int idx = tid; idx < d * d; idx += kPreThreads) {
        const int i = idx / d, j = idx - i * d;
        Wt[j * WS + i] = to_f32(wch[idx]);
      }
    }
    if (K > 0) __syncthreads();

    const int nI2 = d / 4;  // channel pairs (i0, i0+1) in the lower half
    const int ntile = (TT / 4) * nI2;
    for (int idx = tid; idx < ntile; idx += kPreThreads) {
      const int ip = idx % nI2, tq = idx / nI2;
      const int tl0 = tq * 4, i0 = ip * 2, i1 = i0 + half;
      float y[4][4];
      if (full) {
        // y[t, i] = sum_k sum_j W_k[i][j] z[t - k, j]: the halo rows hold t - k
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int k = 0; k < 4; ++k) y[r][k] = 0.f;
        const int chs[4] = {i0, i0 + 1, i1, i1 + 1};
        for (int k = 0; k < K; ++k) {
          const T* wk = wfull + static_cast<int64_t>(k) * d * d;
#pragma unroll 4
          for (int j = 0; j < d; ++j) {
            float zr[4], wv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) zr[r] = to_f32(z[(tl0 + r + HALO - k) * ZC + cb + j]);
#pragma unroll
            for (int c = 0; c < 4; ++c) wv[c] = to_f32(__ldg(wk + chs[c] * d + j));
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int c = 0; c < 4; ++c) y[r][c] = fmaf(zr[r], wv[c], y[r][c]);
          }
        }
      } else if (wch) {
#pragma unroll
        for (int r = 0; r < 4; ++r)
#pragma unroll
          for (int k = 0; k < 4; ++k) y[r][k] = 0.f;
#pragma unroll 8
        for (int j = 0; j < d; ++j) {
          const float4 uu = *reinterpret_cast<const float4*>(u + j * US + tl0);
          const float2 wl = *reinterpret_cast<const float2*>(Wt + j * WS + i0);
          const float2 wh = *reinterpret_cast<const float2*>(Wt + j * WS + i1);
          const float ur[4] = {uu.x, uu.y, uu.z, uu.w};
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            y[r][0] = fmaf(ur[r], wl.x, y[r][0]);
            y[r][1] = fmaf(ur[r], wl.y, y[r][1]);
            y[r][2] = fmaf(ur[r], wh.x, y[r][2]);
            y[r][3] = fmaf(ur[r], wh.y, y[r][3]);
          }
        }
      } else if (K > 0) {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          y[r][0] = u[i0 * US + tl0 + r];
          y[r][1] = u[(i0 + 1) * US + tl0 + r];
          y[r][2] = u[i1 * US + tl0 + r];
          y[r][3] = u[(i1 + 1) * US + tl0 + r];
        }
      } else {
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const T* zr = z + (tl0 + r + HALO) * ZC + cb;
          y[r][0] = to_f32(zr[i0]);
          y[r][1] = to_f32(zr[i0 + 1]);
          y[r][2] = to_f32(zr[i1]);
          y[r][3] = to_f32(zr[i1 + 1]);
        }
      }
      const int ch[4] = {i0, i0 + 1, i1, i1 + 1};
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int tl = tl0 + r, t = t0 + tl;
        if (t >= S) continue;
        const T* zrow = z + (tl + HALO) * ZC;
        if (a.qk_mean == 2) {
          // "self" reading: the mean of the head's own pre-conv value and y
#pragma unroll
          for (int k = 0; k < 4; ++k) y[r][k] = 0.5f * (y[r][k] + to_f32(zrow[cb + ch[k]]));
        } else if (a.qk_mean) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float kp = to_f32(zrow[QC + ch[k]]);
            float qp;
            if (is_q) {
              qp = to_f32(zrow[hh * d + ch[k]]);
            } else {
              qp = 0.f;
              for (int hl = 0; hl < G; ++hl) qp += to_f32(zrow[hl * d + ch[k]]);
              qp /= static_cast<float>(G);
            }
            y[r][k] += 0.5f * (qp + kp);
          }
        }
        if (a.rope_on) {
          const float2 c0 = cs[tl * half + i0], c1 = cs[tl * half + i0 + 1];
          const float a0 = y[r][0], b0 = y[r][2], a1 = y[r][1], b1 = y[r][3];
          y[r][0] = a0 * c0.x - b0 * c0.y;
          y[r][2] = a0 * c0.y + b0 * c0.x;
          y[r][1] = a1 * c1.x - b1 * c1.y;
          y[r][3] = a1 * c1.y + b1 * c1.x;
        }
        T* dst = is_q ? a.q_out + ((static_cast<int64_t>(b) * S + t) * a.Hq + head) * d
                      : a.k_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + t) * d;
        using V2 = typename Vec2<T>::type;
        *reinterpret_cast<V2*>(dst + i0) = Vec2<T>::make(y[r][0], y[r][1]);
        *reinterpret_cast<V2*>(dst + i1) = Vec2<T>::make(y[r][2], y[r][3]);
      }
    }
    if (K > 0) __syncthreads();
  }

  // 4. value-shift: bit-exact gather of the current / previous v~ row (upper
  // half-channels, or the whole head when it is one of the last floor(Hkv / 2)).
  const bool shift_head = a.value_shift == 2 && g >= a.Hkv - a.Hkv / 2;
  constexpr int VEC = 16 / sizeof(T);
  const int nchunk = d / VEC;
  for (int idx = tid; idx < TT * nchunk; idx += kPreThreads) {
    const int tl = idx / nchunk, i = (idx - tl * nchunk) * VEC;
    const int t = t0 + tl;
    if (t >= S) continue;
    const int row = ((a.value_shift == 1 && i >= half) || shift_head) ? tl + HALO - 1 : tl + HALO;
    const uint4 val = *reinterpret_cast<const uint4*>(z + row * ZC + QC + d + i);
    *reinterpret_cast<uint4*>(a.v_out + ((static_cast<int64_t>(b) * a.Hkv + g) * a.kv_cap + t) * d +
                              i) = val;
  }

  // 5. decode state, written by the CTA that holds position S-1 (its rows
  // S-KH .. S-1 are all staged; rows before position 0 are zero).
  if (a.len != nullptr && t0 <= S - 1 && S - 1 < t0 + TT) {
    const int KH = L.KH, Hq = a.Hq, Hkv = a.Hkv;
    for (int r = 0; r < KH; ++r) {
      const T* zrow = z + (S - KH + r - t0 + HALO) * ZC;
      for (int c = tid; c < QC + d; c += kPreThreads) {
        if (c < QC)
          a.hist_q[(static_cast<int64_t>(b) * KH + r) * Hq * d + qcol0 + c] = zrow[c];
        else
          a.hist_k[(static_cast<int64_t>(b) * KH + r) * Hkv * d + g * d + (c - QC)] = zrow[c];
      }
    }
    if (a.v_prev) {
      const T* zrow = z + (S - 1 - t0 + HALO) * ZC;
      for (int i = tid; i < d; i += kPreThreads)
        a.v_prev[static_cast<int64_t>(b) * Hkv * d + g * d + i] = zrow[QC + d + i];
    }
    if (g == 0 && tid == 0) a.len[b] = S;
  }
}

}  // namespace

bool pre_attn_fits(int K, int G, int d, int es, bool has_mix) {
  return pre_layout(8, K, G, d, es, has_mix).bytes <= 227 * 1024;
}

template <typename T>
cudaError_t launch_pre_attn(const PreAttnArgs<T>& a, cudaStream_t stream) {
  if constexpr (std::is_same<T, bf16>::value) {
    if (pre_attn_tc_supported(a)) return launch_pre_attn_tc(a, stream);
  }
  // Positions per CTA: TT * d = 4096 gives exactly one 4x4 register tile per
  // thread in the channel mix; halve TT while the staging does not fit.
  int TT = 4096 / a.d;
  if (TT > 256) TT = 256;
  const int es = sizeof(T);
  const bool has_mix = !a.channel_conv && (a.wq_chan != nullptr || a.wk_chan != nullptr);
  while (TT > 8 && pre_layout(TT, a.K, a.G, a.d, es, has_mix).bytes > 200 * 1024) TT /= 2;
  const PreLayout L = pre_layout(TT, a.K, a.G, a.d, es, has_mix);
  if (L.bytes > 227 * 1024) return cudaErrorInvalidConfiguration;
  auto kernel = a.d == 16 ? pre_attn_kernel<T, 16>
              : a.d == 32 ? pre_attn_kernel<T, 32>
              : a.d == 64 ? pre_attn_kernel<T, 64>
                          : pre_attn_kernel<T, 128>;
  if (a.d != 16 && a.d != 32 && a.d != 64 && a.d != 128) return cudaErrorInvalidValue;
  cudaError_t e = allow_smem(reinterpret_cast<const void*>(kernel),
                                       static_cast<int>(L.bytes));
  if (e != cudaSuccess) return e;
  dim3 grid((a.S + TT - 1) / TT, a.Hkv, a.B);
  kernel<<<grid, kPreThreads, L.bytes, stream>>>(a, TT);
  count_launches(1);
  return cudaGetLastError();
}

template cudaError_t launch_pre_attn<float>(const PreAttnArgs<float>&, cudaStream_t);
template cudaError_t launch_pre_attn<bf16>(const PreAttnArgs<bf16>&, cudaStream_t);

}  // namespace ccgqa
