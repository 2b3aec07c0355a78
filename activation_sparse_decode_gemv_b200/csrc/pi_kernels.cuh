// pi_kernels.cuh -- CUDA-core kernels of the predictor-gated sparse FFN
// decode step (PowerInfer summary page: Summary, second paragraph, a small
// predictor per layer and kernels specialised to single neurons; Interesting
// ideas I4, kernels that work directly on the rows of active neurons).
//
// Per layer and token batch the chain is
//   rmsnorm_kernel     (stacks only)  x fp32 -> u fp16
//   pred_h_kernel      h = P1 u                         (warp per P1 row)
//   pred_s_kernel      s = P2 h + bias, fire iff s > 0, one mask word per
//                      32 neurons and token             (warp per 4 P2 rows)
//   compact_kernel     ascending id lists per token, the union of the
//                      tokens' sets, its per-word prefix (block scan)
//   ffn_gather_kernel  rows of the union: up/gate dot + activation, then
//                      down-projection rows of the live neurons into one
//                      fp32 partial of y per CTA
//   reduce_kernel      y = sum of the partials in CTA order (deterministic,
//                      no atomics), optionally accumulated into y or x.
// Every kernel is launched with programmatic dependent launch: it may start
// while its predecessor drains, prefetches its own weight rows into L2, and
// waits (griddepcontrol.wait) before reading anything the predecessor wrote.
#pragma once

#include "pi_device.cuh"

namespace pi {

// ============================================================== mixed-precision dots
// 8 fp16 weights times 8 fp16 inputs (16 B each) into two fp32 chains with
// the mixed-precision FMA: the product of two fp16 values is exact in fp32,
// so each step equals fmaf((float)w, (float)u, acc) bit for bit, without the
// conversions.
PI_DEV void mdot8(const uint4 &w, const uint4 &u, float &x, float &y) {
  const unsigned ws[4] = {w.x, w.y, w.z, w.w}, us[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %2;\n mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.f16 %0, al, bl, %0;\n fma.rn.f32.f16 %1, ah, bh, %1;\n}\n"
        : "+f"(x), "+f"(y)
        : "r"(ws[k]), "r"(us[k]));
}
// the 8 int4 codes of one 32-bit word (element 2k = low nibble of byte k) as
// four fp16 pairs (q - 8), in element order: 0x6400 | q is the fp16 value
// 1024 + q, and subtracting 1032 is exact
PI_DEV uint4 q8_pairs(uint32_t w) {
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
  uint32_t o[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t t = w >> (8 * k);
    const uint32_t hb = (t & 0xFu) | ((t & 0xF0u) << 12) | 0x64006400u;
    const __half2 v = __hsub2(*reinterpret_cast<const __half2 *>(&hb), off);
    o[k] = *reinterpret_cast<const uint32_t *>(&v);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// ============================================================== rmsnorm
// u_b = fp16(x_b / sqrt(mean(x_b^2) + 1e-6)).  The sum of squares is taken in
// double (each square is exact), the mean is rounded once to float, and the
// remaining steps are single correctly rounded binary32 operations, so the
// fp16 code depends only on x, not on the summation order.
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float *__restrict__ x, int d, __half *__restrict__ u) {
  pdl_wait();
  const int b = blockIdx.x;
  const float *xb = x + (size_t)b * d;
  double ss = 0.0;
  for (int k = threadIdx.x; k < d; k += blockDim.x) {
    const double v = (double)xb[k];
    ss += v * v;
  }
  __shared__ double red[8];
  __shared__ float s_den;
  ss = warp_sum_d(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    const float mean = __double2float_rn(t / (double)d);
    s_den = __fsqrt_rn(__fadd_rn(mean, 1e-6f));
  }
  __syncthreads();
  pdl_launch_dependents();
  const float den = s_den;
  for (int k = threadIdx.x; k < d; k += blockDim.x) u[(size_t)b * d + k] = __float2half_rn(__fdiv_rn(xb[k], den));
}

// ============================================================== predictor, stage 1
// h[t][j] = P1_j . u_t.  Warp per row j; 8 rows per CTA; grid.y = token groups.
template <int NB, int WT>
__global__ void __launch_bounds__(256)
    pred_h_kernel(const void *__restrict__ p1, const void *__restrict__ u, int d, int r, int B, float *__restrict__ h) {
  constexpr int E = Chunk<WT>::elems;
  constexpr int UNR = 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.x * 8 + warp;
  const int t0 = blockIdx.y * NB;
  const size_t rb = (size_t)d * (WT == W_F32 ? 4 : 2);
  const char *row = reinterpret_cast<const char *>(p1) + (size_t)j * rb;
  if (j < r)
    for (size_t off = (size_t)lane * 128; off < rb; off += 32 * 128) l2_prefetch(row + off);
  pdl_wait();
  pdl_launch_dependents();
  if (j >= r) return;
  const int nch = d / E;
  const size_t ub = rb;  // bytes of one token row of u (same element type as P1)
  const char *ubase = reinterpret_cast<const char *>(u) + (size_t)t0 * ub;
  float acc[NB];
#pragma unroll
  for (int t = 0; t < NB; ++t) acc[t] = 0.f;
  for (int c = lane; c < nch; c += 32 * UNR) {
    uint4 w[UNR];
#pragma unroll
    for (int q = 0; q < UNR; ++q)
      if (c + 32 * q < nch) w[q] = ld_stream16(row + (size_t)(c + 32 * q) * 16);
#pragma unroll
    for (int q = 0; q < UNR; ++q)
      if (c + 32 * q < nch) {
#pragma unroll
        for (int t = 0; t < NB; ++t)
          if (t0 + t < B) {
            if constexpr (WT == W_F16) {
              float x = 0.f, y = 0.f;
              mdot8(w[q], ld_keep16(ubase + (size_t)t * ub + (size_t)(c + 32 * q) * 16), x, y);
              acc[t] += x + y;
            } else {
              acc[t] += chunk_dot<WT>(w[q], ubase + (size_t)t * ub, (c + 32 * q) * E);
            }
          }
      }
  }
#pragma unroll
  for (int t = 0; t < NB; ++t) {
    const float v = warp_sum(acc[t]);
    if (lane == 0 && t0 + t < B) h[(size_t)(t0 + t) * r + j] = v;
  }
}

// ============================================================== predictor, stage 2
// dot of a 16-byte predictor chunk (fp32 or fp16) with fp32 h at column c0
template <int WT>
PI_DEV float chunk_dot_h(const uint4 &w, const float *h, int c0);
template <>
PI_DEV float chunk_dot_h<W_F32>(const uint4 &w, const float *h, int c0) {
  const float4 hv = ld_keep_f4(h + c0);
  const float4 wv = *reinterpret_cast<const float4 *>(&w);
  float a = wv.x * hv.x;
  a = fmaf(wv.y, hv.y, a);
  a = fmaf(wv.z, hv.z, a);
  return fmaf(wv.w, hv.w, a);
}
template <>
PI_DEV float chunk_dot_h<W_F16>(const uint4 &w, const float *h, int c0) {
  float wf[8];
  h8_to_f8(w, wf);
  const float4 h0 = ld_keep_f4(h + c0), h1 = ld_keep_f4(h + c0 + 4);
  float a = wf[0] * h0.x;
  a = fmaf(wf[1], h0.y, a);
  a = fmaf(wf[2], h0.z, a);
  a = fmaf(wf[3], h0.w, a);
  a = fmaf(wf[4], h1.x, a);
  a = fmaf(wf[5], h1.y, a);
  a = fmaf(wf[6], h1.z, a);
  return fmaf(wf[7], h1.w, a);
}

// s_i = P2_i . h + bias_i; neuron i fires iff s_i > 0.  One CTA per tile of
// 32 neurons (one mask word per token); warp w owns rows 4w .. 4w+3.
template <int NB, int WT>
__global__ void __launch_bounds__(256)
    pred_s_kernel(const void *__restrict__ p2, const float *__restrict__ h, const float *__restrict__ bias, int f,
                  int r, int B, uint32_t *__restrict__ mask, int nwords) {
  constexpr int E = Chunk<WT>::elems;
  __shared__ uint32_t s_bits[NB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, t0 = blockIdx.y * NB;
  if (threadIdx.x < NB) s_bits[threadIdx.x] = 0u;
  const size_t rb = (size_t)r * (WT == W_F32 ? 4 : 2);
  const int i0 = tile * 32 + warp * 4;
  const char *rows = reinterpret_cast<const char *>(p2) + (size_t)i0 * rb;
#pragma unroll
  for (int q = 0; q < 4; ++q)
    if (i0 + q < f)
      for (size_t off = (size_t)lane * 128; off < rb; off += 32 * 128) l2_prefetch(rows + q * rb + off);
  pdl_wait();
  pdl_launch_dependents();
  const int nch = r / E;
  float acc[4][NB];
#pragma unroll
  for (int q = 0; q < 4; ++q)
#pragma unroll
    for (int t = 0; t < NB; ++t) acc[q][t] = 0.f;
#pragma unroll 2
  for (int c = lane; c < nch; c += 32) {
    uint4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) w[q] = (i0 + q < f) ? ld_stream16(rows + q * rb + (size_t)c * 16) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int t = 0; t < NB; ++t)
      if (t0 + t < B) {
        const float *ht = h + (size_t)(t0 + t) * r;
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q][t] += chunk_dot_h<WT>(w[q], ht, c * E);
      }
  }
  uint32_t fired[NB];
#pragma unroll
  for (int t = 0; t < NB; ++t) fired[t] = 0u;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float bq = (i0 + q < f) ? bias[i0 + q] : 0.f;
#pragma unroll
    for (int t = 0; t < NB; ++t) {
      const float s = warp_sum(acc[q][t]) + bq;
      if (i0 + q < f && s > 0.f) fired[t] |= 1u << (warp * 4 + q);
    }
  }
  __syncthreads();
  if (lane == 0) {
#pragma unroll
    for (int t = 0; t < NB; ++t)
      if (fired[t]) atomicOr(&s_bits[t], fired[t]);
  }
  __syncthreads();
  if (threadIdx.x < NB && t0 + (int)threadIdx.x < B) mask[(size_t)(t0 + threadIdx.x) * nwords + tile] = s_bits[threadIdx.x];
}

// ============================================================== compaction
// CTA b < B: token b's ascending id list (only when idx != nullptr) and count;
// CTA B: union mask words, exclusive prefix of their popcounts (uprefix has
// nwords + 1 entries), the ascending union list and its length.
__global__ void __launch_bounds__(1024)
    compact_kernel(const uint32_t *__restrict__ mask, int nwords, int idx_stride, int B, int32_t *__restrict__ idx,
                   int32_t *__restrict__ count, uint32_t *__restrict__ uwords, int32_t *__restrict__ uprefix,
                   int32_t *__restrict__ ulist, int32_t *__restrict__ ucount) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.x;
  const bool is_union = (b == B);
  if (!is_union && idx == nullptr && count == nullptr) return;
  __shared__ int32_t s_warp[32];
  __shared__ int32_t s_carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  if (threadIdx.x == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < nwords; base += blockDim.x) {
    const int w = base + threadIdx.x;
    uint32_t word = 0u;
    if (w < nwords) {
      if (!is_union) {
        word = mask[(size_t)b * nwords + w];
      } else {
        // 8 independent loads in flight per round
        for (int t0 = 0; t0 < B; t0 += 8) {
          uint32_t v[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v[k] = t0 + k < B ? mask[(size_t)(t0 + k) * nwords + w] : 0u;
#pragma unroll
          for (int k = 0; k < 8; ++k) word |= v[k];
        }
        uwords[w] = word;
      }
    }
    const int c = __popc(word);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int v = lane < nwarp ? s_warp[lane] : 0;
      int inc = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int q = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += q;
      }
      s_warp[lane] = inc - v;  // exclusive prefix of warp totals
    }
    __syncthreads();
    const int carry = s_carry;
    int pos = carry + s_warp[warp] + incl - c;
    if (is_union && w < nwords) uprefix[w] = pos;
    int32_t *out = is_union ? ulist : (idx ? idx + (size_t)b * idx_stride : nullptr);
    if (out) {
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1u;
        out[pos++] = w * 32 + bit;
      }
    }
    __syncthreads();
    if (threadIdx.x == blockDim.x - 1) s_carry = carry + s_warp[warp] + incl;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (is_union) {
      *ucount = s_carry;
      uprefix[nwords] = s_carry;
    } else if (count) {
      count[b] = s_carry;
    }
  }
}

// caller id lists -> mask words (mask zeroed beforehand).  Lists are sets:
// order and repeats do not matter; ids outside [0, f) and counts outside
// [0, f] are skipped / clamped and flag the device status.
__global__ void __launch_bounds__(256)
    idx_to_mask_kernel(const int32_t *__restrict__ idx, const int32_t *__restrict__ count, int f,
                       uint32_t *__restrict__ mask, int nwords, int *__restrict__ status) {
  pdl_wait();
  pdl_launch_dependents();
  const int b = blockIdx.y;
  int n = count[b];
  if (n < 0 || n > f) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(status, kStatusDeviceArg);
    n = n < 0 ? 0 : f;
  }
  for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n; k += gridDim.x * blockDim.x) {
    const int i = idx[(size_t)b * f + k];
    if ((unsigned)i >= (unsigned)f) {
      set_status(status, kStatusDeviceArg);
      continue;
    }
    atomicOr(&mask[(size_t)b * nwords + (i >> 5)], 1u << (i & 31));
  }
}

// ============================================================== gather FFN
struct FfnArgs {
  const void *w_up, *w_gate, *w_down_t;
  const __half *s_up, *s_gate, *s_down_t;
  const float *b_up;
  const void *u;  // [B x d], fp32 for W_F32 else fp16
  int d, f, B;
  const uint32_t *mask;
  int nwords;
  const int32_t *ulist, *ucount, *uprefix;
  int hot_dense, H;  // H % 32 == 0
  float *partial;    // [G x B x d]
};

// number of neurons of the virtual list processed by the grid, and the
// half-open range of CTA c; the reducer uses the same formula
PI_DEV int virtual_len(const int32_t *ucount, const int32_t *uprefix, int hot_dense, int H) {
  const int U = *ucount;
  return hot_dense ? H + (U - uprefix[H >> 5]) : U;
}
PI_DEV int chunk_begin(int c, int V, int G) { return (int)(((long long)c * V) / G); }

// one warp: dots of row i of NR matrices (W[0], W[1]: up and gate) with the
// NB tokens of this group; all lanes get the sums.  fp16 and int4 weights
// multiply the fp16 tokens with the mixed-precision FMA (no conversions);
// the rows of both matrices stream in the same loop (8 loads per lane in
// flight in total).
template <int NB, int WT, int NR>
PI_DEV void row_dots(const void *const *W, const __half *const *S, int i, const void *u, int d, int B, int t0,
                     int lane, float (&out)[NR][NB]) {
  constexpr int E = Chunk<WT>::elems;
  constexpr int UNR = 8 / NR;  // 8 loads per lane in flight over the NR rows
  const size_t rb = WT == W_F32 ? (size_t)d * 4 : WT == W_F16 ? (size_t)d * 2 : (size_t)d / 2;
  const size_t ub = WT == W_F32 ? (size_t)d * 4 : (size_t)d * 2;
  const char *ubase = reinterpret_cast<const char *>(u) + (size_t)t0 * ub;
  const int nch = d / E;
#pragma unroll
  for (int m = 0; m < NR; ++m)
#pragma unroll
    for (int t = 0; t < NB; ++t) out[m][t] = 0.f;
  for (int c = lane; c < nch; c += 32 * UNR) {
    uint4 w[NR][UNR];
#pragma unroll
    for (int m = 0; m < NR; ++m) {
      const char *row = reinterpret_cast<const char *>(W[m]) + (size_t)i * rb;
#pragma unroll
      for (int q = 0; q < UNR; ++q)
        if (c + 32 * q < nch) w[m][q] = ld_stream16(row + (size_t)(c + 32 * q) * 16);
    }
#pragma unroll
    for (int q = 0; q < UNR; ++q) {
      const int cc = c + 32 * q;
      if (cc >= nch) continue;
#pragma unroll
      for (int m = 0; m < NR; ++m) {
        if constexpr (WT == W_F32) {
#pragma unroll
          for (int t = 0; t < NB; ++t)
            if (t0 + t < B) out[m][t] += chunk_dot<WT>(w[m][q], ubase + (size_t)t * ub, cc * E);
        } else if constexpr (WT == W_F16) {
#pragma unroll
          for (int t = 0; t < NB; ++t)
            if (t0 + t < B) {
              float x = 0.f, y = 0.f;
              mdot8(w[m][q], ld_keep16(ubase + (size_t)t * ub + (size_t)cc * 16), x, y);
              out[m][t] += x + y;
            }
        } else {
          // one chunk = one 32-element group: (q - 8) pairs, then the group scale
          const float sc = __half2float(S[m][(size_t)i * (d / 32) + cc]);
          const uint4 p0 = q8_pairs(w[m][q].x), p1 = q8_pairs(w[m][q].y), p2 = q8_pairs(w[m][q].z),
                      p3 = q8_pairs(w[m][q].w);
#pragma unroll
          for (int t = 0; t < NB; ++t)
            if (t0 + t < B) {
              const char *uc = ubase + (size_t)t * ub + (size_t)cc * 64;
              float x = 0.f, y = 0.f;
              mdot8(p0, ld_keep16(uc), x, y);
              mdot8(p1, ld_keep16(uc + 16), x, y);
              mdot8(p2, ld_keep16(uc + 32), x, y);
              mdot8(p3, ld_keep16(uc + 48), x, y);
              out[m][t] = fmaf(sc, x + y, out[m][t]);
            }
        }
      }
    }
  }
#pragma unroll
  for (int m = 0; m < NR; ++m)
#pragma unroll
    for (int t = 0; t < NB; ++t) out[m][t] = warp_sum(out[m][t]);
}

// 8 consecutive elements (column group g) of W2T row i, as floats
template <int WT>
PI_DEV void load_group(const void *W, const __half *S, int i, int d, int g, float o[8]);
template <>
PI_DEV void load_group<W_F32>(const void *W, const __half *, int i, int d, int g, float o[8]) {
  const char *p = reinterpret_cast<const char *>(W) + ((size_t)i * d + (size_t)g * 8) * 4;
  const uint4 a = ld_stream16(p), b = ld_stream16(p + 16);
  const float *fa = reinterpret_cast<const float *>(&a), *fb = reinterpret_cast<const float *>(&b);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[k] = fa[k];
    o[4 + k] = fb[k];
  }
}
template <>
PI_DEV void load_group<W_F16>(const void *W, const __half *, int i, int d, int g, float o[8]) {
  h8_to_f8(ld_stream16(reinterpret_cast<const char *>(W) + ((size_t)i * d + (size_t)g * 8) * 2), o);
}
template <>
PI_DEV void load_group<W_INT4>(const void *W, const __half *S, int i, int d, int g, float o[8]) {
  const uint32_t q = ld_stream4(reinterpret_cast<const char *>(W) + (size_t)i * (d / 2) + (size_t)g * 4);
  const float sc = __half2float(S[(size_t)i * (d / 32) + (g >> 2)]);
  q8_to_f8(q, o);
#pragma unroll
  for (int k = 0; k < 8; ++k) o[k] *= sc;
}

// CTA c handles the neurons [chunk_begin(c), chunk_begin(c+1)) of the virtual
// list (hot prefix rows 0..H-1 first in dense mode, then the union's tail
// ids), in sub-chunks of CH: up/gate dots by warps, then the down-projection
// rows of the neurons with a nonzero value, accumulated per column group by
// each thread; the CTA writes one partial of y.
template <int NB, int WT, int ACT, int GPT>
__global__ void __launch_bounds__(512) ffn_gather_kernel(FfnArgs a) {
  constexpr int CH = 64;
  __shared__ int32_t s_nid[CH];
  __shared__ uint32_t s_memb[CH];
  __shared__ float s_a[NB][CH];
  __shared__ int32_t s_live[CH];
  __shared__ int s_nlive;
  const int G = gridDim.x, c = blockIdx.x, t0 = blockIdx.y * NB;
  const int nwarps = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = a.d, B = a.B;
  pdl_wait();
  pdl_launch_dependents();
  const int V = virtual_len(a.ucount, a.uprefix, a.hot_dense, a.H);
  const int pb = chunk_begin(c, V, G), pe = chunk_begin(c + 1, V, G);
  const int ngroups = d / 8;
  const int upre_h = a.hot_dense ? a.uprefix[a.H >> 5] : 0;

  float acc[GPT][NB][8];
#pragma unroll
  for (int q = 0; q < GPT; ++q)
#pragma unroll
    for (int t = 0; t < NB; ++t)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[q][t][e] = 0.f;

  for (int base = pb; base < pe; base += CH) {
    const int n = min(CH, pe - base);
    if ((int)threadIdx.x < n) {
      const int p = base + threadIdx.x;
      const int i = a.hot_dense ? (p < a.H ? p : a.ulist[upre_h + (p - a.H)]) : a.ulist[p];
      uint32_t m = 0u;
#pragma unroll
      for (int t = 0; t < NB; ++t)
        if (t0 + t < B) m |= ((a.mask[(size_t)(t0 + t) * a.nwords + (i >> 5)] >> (i & 31)) & 1u) << t;
      s_nid[threadIdx.x] = i;
      s_memb[threadIdx.x] = m;
    }
    __syncthreads();
    // up / gate rows: one warp per neuron
    for (int k = warp; k < n; k += nwarps) {
      const int i = s_nid[k];
      const uint32_t m = s_memb[k];
      const bool dense_row = a.hot_dense && i < a.H;
      float av[NB];
      if (m == 0u && !dense_row) {
#pragma unroll
        for (int t = 0; t < NB; ++t) av[t] = 0.f;
      } else if constexpr (ACT == ACT_SWIGLU) {
        const void *Ws[2] = {a.w_up, a.w_gate};
        const __half *Ss[2] = {a.s_up, a.s_gate};
        float v[2][NB];
        row_dots<NB, WT, 2>(Ws, Ss, i, a.u, d, B, t0, lane, v);
#pragma unroll
        for (int t = 0; t < NB; ++t) av[t] = ((m >> t) & 1u) ? silu(v[1][t]) * v[0][t] : 0.f;
      } else {
        const void *Ws[1] = {a.w_up};
        const __half *Ss[1] = {a.s_up};
        float v[1][NB];
        row_dots<NB, WT, 1>(Ws, Ss, i, a.u, d, B, t0, lane, v);
        const float bi = a.b_up[i];
#pragma unroll
        for (int t = 0; t < NB; ++t) av[t] = ((m >> t) & 1u) ? fmaxf(v[0][t] + bi, 0.f) : 0.f;
      }
      if (lane == 0) {
#pragma unroll
        for (int t = 0; t < NB; ++t) s_a[t][k] = av[t];
      }
    }
    __syncthreads();
    // live list: neurons contributing a nonzero value to some token
    if (warp == 0) {
      int nl = 0;
      for (int k0 = 0; k0 < n; k0 += 32) {
        const int k = k0 + lane;
        bool live = false;
        if (k < n) {
#pragma unroll
          for (int t = 0; t < NB; ++t) live |= (s_a[t][k] != 0.f);
        }
        const uint32_t bal = __ballot_sync(0xffffffffu, live);
        if (live) s_live[nl + __popc(bal & ((1u << lane) - 1u))] = k;
        nl += __popc(bal);
      }
      if (lane == 0) s_nlive = nl;
    }
    __syncthreads();
    const int nl = s_nlive;
    // down-projection rows, accumulated per column group
#pragma unroll
    for (int q = 0; q < GPT; ++q) {
      const int g = threadIdx.x + q * blockDim.x;
      if (g < ngroups) {
        for (int kk = 0; kk < nl; kk += 4) {
          float w[4][8];
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (kk + j < nl) load_group<WT>(a.w_down_t, a.s_down_t, s_nid[s_live[kk + j]], d, g, w[j]);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (kk + j < nl) {
              const int k = s_live[kk + j];
#pragma unroll
              for (int t = 0; t < NB; ++t) {
                const float av = s_a[t][k];
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[q][t][e] = fmaf(av, w[j][e], acc[q][t][e]);
              }
            }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int q = 0; q < GPT; ++q) {
    const int g = threadIdx.x + q * blockDim.x;
    if (g < ngroups) {
#pragma unroll
      for (int t = 0; t < NB; ++t)
        if (t0 + t < B) {
          float4 *dst = reinterpret_cast<float4 *>(a.partial + ((size_t)c * B + t0 + t) * d + (size_t)g * 8);
          dst[0] = make_float4(acc[q][t][0], acc[q][t][1], acc[q][t][2], acc[q][t][3]);
          dst[1] = make_float4(acc[q][t][4], acc[q][t][5], acc[q][t][6], acc[q][t][7]);
        }
    }
  }
}

// ============================================================== reduction
// out[e] (= or +=) sum over all CTAs c of partial[c][e] (CTAs without neurons
// wrote zeros).  A CTA covers 32 consecutive elements; thread (e, g) sums the
// partials c = g, g + 8, ... in increasing c, then the 8 group sums are added
// in increasing g: a fixed order, so the result is deterministic, and no
// atomics are used.
__global__ void __launch_bounds__(256)
    reduce_kernel(const float *__restrict__ partial, int G, int n_elem, float *__restrict__ out, int accumulate) {
  __shared__ float s_part[8][33];
  pdl_wait();
  pdl_launch_dependents();
  const int el = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int e = blockIdx.x * 32 + el;
  float s = 0.f;
  if (e < n_elem) {
    int c = g;
    for (; c + 24 < G; c += 32) {
      const float a0 = partial[(size_t)c * n_elem + e], a1 = partial[(size_t)(c + 8) * n_elem + e];
      const float a2 = partial[(size_t)(c + 16) * n_elem + e], a3 = partial[(size_t)(c + 24) * n_elem + e];
      s += a0;
      s += a1;
      s += a2;
      s += a3;
    }
    for (; c < G; c += 8) s += partial[(size_t)c * n_elem + e];
  }
  s_part[g][el] = s;
  __syncthreads();
  if (g == 0 && e < n_elem) {
    float t = s_part[0][el];
#pragma unroll
    for (int k = 1; k < 8; ++k) t += s_part[k][el];
    out[e] = accumulate ? out[e] + t : t;
  }
}

}  // namespace pi
