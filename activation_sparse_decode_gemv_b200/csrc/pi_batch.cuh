// pi_batch.cuh -- the decode step of a token batch of 2..8 with fp16 weights
// (PowerInfer summary page: Summary, per-layer predictor and neuron-aware
// sparse operators; Interesting ideas I4, kernels that read only the rows of
// the active neurons), as two persistent kernels per layer:
// pred_batch_kernel (steps 1-2, at the end of this file) and
// ffn_batch_kernel (steps 2-4 over the union of the tokens' sets).
//
// Grid: one CTA per SM (all co-resident; each kernel's one grid-wide wait is
// bounded).  The products are small matrix products with the batch as N = 8
// columns, so they run on the tensor cores (mma.sync m16n8k16, fp16 inputs,
// fp32 accumulation); the work is bound by HBM, and the tensor cores only
// keep the instruction count per weight byte low.
//
// ffn_batch_kernel:
// Union.  Every CTA scans the union words (the OR of the tokens' mask
// words) itself: block prefix of their popcounts, so a list position maps to
// its neuron id by a binary search and a bit select.  The list is the hot
// prefix densely (dense mode), then the union's other neurons ascending.
//
// Step 3 (up / gate + activation).  CTA c takes the list positions
// [list_begin(c), list_begin(c + 1)), in groups of 16 neurons (the MMA's M).
// A unit is 64 elements of the 16 rows of a group.  The weight rows go from
// HBM straight into registers: lane (g, q) of a warp loads the 32 bytes at
// elements 16q .. 16q + 15 of rows g and g + 8 (one 256-bit load each, so the
// four lanes of a row read its whole 128-byte line in one instruction; half
// lines per instruction were measured to cost HBM more than half its
// bandwidth).  Those are A fragments once the K order inside the unit is
// permuted the same way for the token operand (a dot product does not depend
// on the order of its terms).  The tokens sit in shared memory.  Warp w takes
// the units w, w + 16, ... of every group, so the 16 warps read one
// contiguous 2 KB run of each of the group's rows together; each leaves its
// partial of the group in shared memory (double-buffered by group) and, after
// the group's barrier, the CTA adds them in warp order.  The activation a
// (zero for tokens that did not predict the neuron) is stored as two fp16
// parts, a_hi = fp16(a) and a_lo = fp16(a - a_hi), so step 4 carries a to
// about 22 bits.  The CTA also writes its positions' ids into the union list.
//
// Step 4 (down).  y^T [d x 8] = W2T^T [d x list] * a [list x 8].  A unit is a
// tile of 64 columns of y times 16 list positions; units are ordered tile by
// tile and split into G contiguous spans (stream-K over CTAs), so every CTA
// does the same amount of work.  Inside a CTA the warps take the units of a
// tile in turn (an incremental cursor walks them: per-unit bookkeeping was
// measured to bound this stream before) and each keeps its own ring of 3
// shared-memory stages filled with cp.async (16-byte copies, XOR-swizzled so
// that ldmatrix.trans reads them without bank conflicts); the activations of
// the unit's positions ride in the same stage.  A tile covered by one CTA is
// written to y directly; a tile split between CTAs is finished by the last
// CTA to arrive (per-tile counter), which adds the pieces in CTA order, so
// the result does not depend on timing.  Counters reset themselves.
//
// Shared memory stays near 150 KB: register loads need L1 room (a streaming
// read was measured to drop from 6.3 to 4.5 TB/s with 200 KB of shared
// memory per SM).
#pragma once

#include <cuda.h>

#include "pi_device.cuh"
#include "pi_fused.cuh"

namespace pi {
namespace batch {

using fused::grid_barrier;
using fused::mma_16816;
using fused::smem_u32;

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kTok = 8;          // token columns (batches of 2..8; rows past B are zero)
constexpr int kKStep = 64;       // elements of one step-3 unit
constexpr int kTileCols = 64;    // columns of y per step-4 tile
constexpr int kPosStep = 16;     // list positions per step-4 unit
constexpr int kStages = 3;       // step-4 stages per warp (2 units in flight; shared memory is kept
                                 // small, since register loads need L1 room)
constexpr int kRowBytes = kTileCols * 2;
constexpr int kStageBytes = kPosStep * kRowBytes + 2 * kTok * kPosStep * 2;  // rows + a_hi + a_lo
constexpr int kMaxLoc = 512;     // list positions one CTA takes in step 3
constexpr int kMaxTiles = 192;   // step-4 tiles (d <= 12288)
constexpr int kMaxWords = 1024;  // 32-neuron words of the union (d_ffn <= 32768)
constexpr int kPieceFloats = kTileCols * kTok;
constexpr unsigned long long kWaitNs = 2000000000ull;

struct Args {
  const void *w_up, *w_gate, *w_down_t;
  const float *b_up;
  const __half *u;  // [B x d] fp16
  int d, f, B;
  const uint32_t *mask;    // [B x nwords] per-token mask words
  const uint32_t *uwords;  // [nwords] their OR (the union)
  int nwords;
  int32_t *ulist;  // union list, written here: each CTA its own positions
  int hot_dense, H;
  __half *a_hi, *a_lo;  // [kTok x a_stride] activations by list position
  int a_stride;
  float *part;     // [G x 2 x kPieceFloats] pieces of split tiles
  unsigned *ctr;   // [d / kTileCols] arrival counters, zero between launches
  unsigned *bar;   // grid-barrier word
  float *out;      // [B x d]
  int accumulate;  // out += y instead of out = y
  int *status;
  unsigned long long wait_ns;
};

// dynamic shared memory: step 3 (tokens + warp partials) and step 4 (stages +
// tile partials) use the same bytes, one after the other
inline __host__ __device__ size_t step3_bytes(int d, int nmat) {
  return (size_t)kTok * (2 * (size_t)d + 16) + (size_t)2 * kWarps * nmat * 128 * 4;
}
inline __host__ __device__ size_t step4_bytes() {
  return (size_t)kWarps * kStages * kStageBytes;
}
inline __host__ __device__ size_t smem_bytes(int d, int nmat) {
  const size_t a = step3_bytes(d, nmat), b = step4_bytes();
  return a > b ? a : b;
}

// ---------------------------------------------------------------- PTX helpers
PI_DEV void ldmatrix_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// 32 bytes (32-byte aligned) of a weight row, read once: bypass L1.
// Volatile, so the load is issued where it is written (ahead of its use, or
// before the grid-dependency wait) instead of being sunk to its first use.
PI_DEV void ld_stream32(const void *p, uint4 &lo, uint4 &hi) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x), "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
      : "l"(p));
}
PI_DEV void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
PI_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
PI_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// position of the k-th (0-based) set bit of w (k < popc(w)): halve the
// window by the popcount of its low half, five times
PI_DEV int select_bit(uint32_t w, int k) {
  int pos = 0;
#pragma unroll
  for (int width = 16; width >= 1; width >>= 1) {
    const int c = __popc(w & ((1u << width) - 1u));
    if (k >= c) {
      k -= c;
      pos += width;
      w >>= width;
    }
  }
  return pos;
}
PI_DEV void st_shared_zero16(uint32_t dst) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(dst), "r"(0u) : "memory");
}

// first list position of CTA c (the same split as the CUDA-core gather
// kernel)
PI_DEV int list_begin(int c, int V, int G) { return (int)(((long long)c * V) / G); }

// step-4 span of CTA c: units [span_lo(c), span_lo(c + 1)) of W
PI_DEV long long span_lo(long long W, int c, int G) { return W * c / G; }
// the CTA whose span holds unit x (the largest c with span_lo(c) <= x)
PI_DEV int span_owner(long long W, long long x, int G) { return (int)(((x + 1) * G + W - 1) / W) - 1; }

template <int ACT>
__global__ void __launch_bounds__(kThreads, 1) ffn_batch_kernel(const __grid_constant__ Args a) {
  constexpr int NM = ACT == ACT_SWIGLU ? 2 : 1;
  constexpr int PD = ACT == ACT_SWIGLU ? 2 : 3;  // step-3 units in flight per warp
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int ids_s[kMaxLoc];
  __shared__ uint32_t memb_s[kMaxLoc];
  __shared__ float bias_s[kMaxLoc];
  __shared__ int last_s;
  __shared__ uint32_t uw_s[kMaxWords];
  __shared__ int pre_s[kMaxWords + 1];  // exclusive prefix of the union words' popcounts
  __shared__ int wsum_s[kWarps];
  __shared__ int pro_ids_s[kWarps][kStages][kPosStep];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, B = a.B;
  const size_t rb = (size_t)d * 2;

  pdl_wait();
  // the tokens into shared memory (rows B..7 zero), in flight during the
  // union scan; cp.async, so the copy needs no registers
  const int upitch = d + 8;  // halves; rows 16 bytes apart modulo 128 (conflict-free fragment reads)
  __half *u_s = reinterpret_cast<__half *>(smem);
  {
    const int dch = d / 8;
    for (int k = tid; k < kTok * dch; k += kThreads) {
      const int t = k / dch, e = k - t * dch;
      const uint32_t dst = smem_u32(u_s + (size_t)t * upitch + (size_t)e * 8);
      if (t < B)
        cp_async16(dst, a.u + (size_t)t * d + (size_t)e * 8);
      else
        st_shared_zero16(dst);
    }
    cp_async_commit();
  }
  // ---- the union: every CTA scans the union words itself (same result in
  // every CTA), so no separate compaction runs before this kernel
  const int nw = a.nwords;
  {
    uint32_t w0 = 0u, w1 = 0u;
    if (2 * tid < nw) w0 = a.uwords[2 * tid];
    if (2 * tid + 1 < nw) w1 = a.uwords[2 * tid + 1];
    if (2 * tid < nw) uw_s[2 * tid] = w0;
    if (2 * tid + 1 < nw) uw_s[2 * tid + 1] = w1;
    const int c0 = __popc(w0), cnt = c0 + __popc(w1);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) wsum_s[warp] = incl;
    __syncthreads();
    int base = 0;
    for (int w = 0; w < warp; ++w) base += wsum_s[w];
    const int ex = base + incl - cnt;
    if (2 * tid < nw) pre_s[2 * tid] = ex;
    if (2 * tid + 1 < nw) pre_s[2 * tid + 1] = ex + c0;
    if (tid == kThreads - 1) pre_s[nw] = base + incl;
    __syncthreads();
  }
  const int U = pre_s[nw];
  const int upre_h = a.hot_dense ? pre_s[a.H >> 5] : 0;
  const int V = a.hot_dense ? a.H + (U - upre_h) : U;
  // union index of list position p (-1: a dense hot-prefix row, id p)
  auto uidx = [&](int p) -> int { return a.hot_dense ? (p < a.H ? -1 : upre_h + (p - a.H)) : p; };
  // neuron id of union index x, from the scan: binary search, then the bit
  auto id_of_uidx = [&](int x) -> int {
    int lo = 0, hi = nw;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (pre_s[mid] <= x) lo = mid; else hi = mid;
    }
    return lo * 32 + select_bit(uw_s[lo], x - pre_s[lo]);
  };
  auto vid_local = [&](int p) -> int {
    const int x = uidx(p);
    return x < 0 ? p : id_of_uidx(x);
  };
  // after the grid-wide wait: the list written by the CTAs in step 3 (no
  // line of it is read by this SM before that wait, so L1 holds no stale copy)
  auto vid = [&](int p) -> int {
    const int x = uidx(p);
    return x < 0 ? p : a.ulist[x];
  };

  // ---- step-4 spans (known once the list length is): CTA c owns units
  // [u0, u1) of the W = (d / 64) x S (tile, 16-position step) units
  const int ntiles = d / kTileCols;
  const int S = (V + kPosStep - 1) / kPosStep;
  const long long W = (long long)ntiles * S;
  const long long u0 = span_lo(W, c, G), u1 = span_lo(W, c + 1, G);
  const int ta = u0 < u1 ? (int)(u0 / S) : 0, tb = u0 < u1 ? (int)((u1 - 1) / S) : -1;
  // units of tile t in this CTA's span: steps [sa, sb)
  auto tile_steps = [&](int t, int &sa, int &sb) {
    const long long lo = (long long)t * S, hi = lo + S;
    sa = (int)((u0 > lo ? u0 : lo) - lo);
    sb = (int)((u1 < hi ? u1 : hi) - lo);
  };
  // warp w takes the steps sa + w, sa + w + 16, ... of each tile
  auto warp_count = [&](int t, int w) {
    int sa, sb;
    tile_steps(t, sa, sb);
    return sb - sa > w ? (sb - sa - w + kWarps - 1) / kWarps : 0;
  };
  // k-th unit of warp w -> (tile, step); false past its last unit
  auto unit_of_w = [&](int k, int w, int &t, int &s) -> bool {
    for (t = ta; t <= tb; ++t) {
      const int n = warp_count(t, w);
      if (k < n) {
        int sa, sb;
        tile_steps(t, sa, sb);
        s = sa + w + k * kWarps;
        return true;
      }
      k -= n;
    }
    return false;
  };
  // list ids of the first kStages units of every warp (the ones issued before
  // the grid-wide wait, when the list written in step 3 is not complete)
  for (int e = tid; e < kWarps * kStages * kPosStep; e += kThreads) {
    const int w = e / (kStages * kPosStep), k = (e / kPosStep) % kStages, row = e % kPosStep;
    int t, s, id = -1;
    if (unit_of_w(k, w, t, s)) {
      const int p = s * kPosStep + row;
      if (p < V) id = vid_local(p);
    }
    pro_ids_s[w][k][row] = id;
  }

  // ================================================================ step 3
  const int pb = list_begin(c, V, G), pe = list_begin(c + 1, V, G);
  const int nloc = pe - pb;
  float *red = reinterpret_cast<float *>(smem + (size_t)kTok * upitch * 2);
  {
    for (int k = tid; k < nloc; k += kThreads) {
      const int x = uidx(pb + k);
      const int i = x < 0 ? pb + k : id_of_uidx(x);
      if (x >= 0) a.ulist[x] = i;
      uint32_t m = 0u;
      for (int t = 0; t < B; ++t) m |= ((a.mask[(size_t)t * a.nwords + (i >> 5)] >> (i & 31)) & 1u) << t;
      ids_s[k] = i;
      memb_s[k] = m;
      if (ACT == ACT_RELU) bias_s[k] = a.b_up[i];
    }
  }
  cp_async_wait<0>();  // the tokens
  __syncthreads();

  const int ns = d / kKStep;
  const int ng = (nloc + 15) >> 4;
  // warp w takes the steps w, w + 16, ... of every group, so the 16 warps
  // read one contiguous 2 KB run of each of the group's rows at a time
  const int per = ns > warp ? (ns - warp + kWarps - 1) / kWarps : 0;
  const int nu = ng * per;  // this warp's units
  {
    struct Buf {
      uint4 w[NM][4];  // [matrix][row g elements 0-7, 8-15, row g+8 elements 0-7, 8-15] of this lane's 16
    };
    // load cursor: group lj, step index li; the group's row pointers are
    // looked up once per group (integer work per unit stays small)
    int lj = -1, li = per;
    const char *rp0[NM], *rp1[NM];
    auto load = [&](Buf &bf) {
      if (li == per) {
        li = 0;
        ++lj;
        const int r0 = 16 * lj + g, r1 = r0 + 8;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const char *W = reinterpret_cast<const char *>(m == 0 ? a.w_up : a.w_gate);
          rp0[m] = r0 < nloc ? W + (size_t)ids_s[r0] * rb + (size_t)q * 32 : nullptr;
          rp1[m] = r1 < nloc ? W + (size_t)ids_s[r1] * rb + (size_t)q * 32 : nullptr;
        }
      }
      const size_t off = (size_t)(warp + kWarps * li) * (kKStep * 2);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        if (rp0[m])
          ld_stream32(rp0[m] + off, bf.w[m][0], bf.w[m][1]);
        else
          bf.w[m][0] = bf.w[m][1] = make_uint4(0u, 0u, 0u, 0u);
        if (rp1[m])
          ld_stream32(rp1[m] + off, bf.w[m][2], bf.w[m][3]);
        else
          bf.w[m][2] = bf.w[m][3] = make_uint4(0u, 0u, 0u, 0u);
      }
      ++li;
    };
    float acc[NM][4];
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][e] = 0.f;
    // group j's partials: red[j % 2][warp][matrix][lane * 4 + e]
    auto flush = [&](int j) {
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        float *dst = red + ((size_t)(((j & 1) * kWarps + warp) * NM + m) * 128) + lane * 4;
        *reinterpret_cast<float4 *>(dst) = make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[m][e] = 0.f;
      }
    };
    // after group j's barrier: the sums over the warps in warp order,
    // activation, membership; a by list position
    auto reduce_group = [&](int j) {
      if (tid < 128) {
        const int rm = tid >> 3, t = tid & 7, p = 16 * j + rm;
        if (p < nloc) {
          const int ln = (rm & 7) * 4 + (t >> 1), e = (t & 1) + ((rm >> 3) << 1);
          float x[NM];
#pragma unroll
          for (int m = 0; m < NM; ++m) x[m] = 0.f;
#pragma unroll 4
          for (int w = 0; w < kWarps; ++w)
#pragma unroll
            for (int m = 0; m < NM; ++m) x[m] += red[(size_t)(((j & 1) * kWarps + w) * NM + m) * 128 + ln * 4 + e];
          float av = 0.f;
          if ((memb_s[p] >> t) & 1u) {
            if constexpr (ACT == ACT_RELU)
              av = fmaxf(x[0] + bias_s[p], 0.f);
            else
              av = silu(x[1]) * x[0];
          }
          const __half hi = __float2half_rn(av);
          const __half lo = __float2half_rn(av - __half2float(hi));
          a.a_hi[(size_t)t * a.a_stride + pb + p] = hi;
          a.a_lo[(size_t)t * a.a_stride + pb + p] = lo;
        }
      }
    };
    int cj = 0, ci = 0;  // compute cursor: group, step index
    auto compute = [&](const Buf &bf) {
      const int j = cj, i = ci, s = warp + kWarps * i;
      if (++ci == per) {
        ci = 0;
        ++cj;
      }
      // token g's elements 16q .. 16q + 15 of the unit, the same K order as the rows
      const __half *ur = u_s + (size_t)g * upitch + (size_t)s * kKStep + q * 16;
      const uint4 ub0 = *reinterpret_cast<const uint4 *>(ur), ub1 = *reinterpret_cast<const uint4 *>(ur + 8);
#pragma unroll
      for (int m = 0; m < NM; ++m) {
        const uint4 &x0 = bf.w[m][0], &x1 = bf.w[m][1], &y0 = bf.w[m][2], &y1 = bf.w[m][3];
        {
          const uint32_t A[4] = {x0.x, y0.x, x0.y, y0.y};
          mma_16816(acc[m], A, ub0.x, ub0.y);
        }
        {
          const uint32_t A[4] = {x0.z, y0.z, x0.w, y0.w};
          mma_16816(acc[m], A, ub0.z, ub0.w);
        }
        {
          const uint32_t A[4] = {x1.x, y1.x, x1.y, y1.y};
          mma_16816(acc[m], A, ub1.x, ub1.y);
        }
        {
          const uint32_t A[4] = {x1.z, y1.z, x1.w, y1.w};
          mma_16816(acc[m], A, ub1.z, ub1.w);
        }
      }
      if (i == per - 1) {  // this warp's last step of group j
        flush(j);
        __syncthreads();
        reduce_group(j);
      }
    };
    if (per == 0) {  // a warp with no step (d < 1024): zeros, and the same barriers
      for (int j = 0; j < ng; ++j) {
        flush(j);
        __syncthreads();
        reduce_group(j);
      }
    } else {
      // loads run PD - 1 units ahead of the MMAs, across group ends
      Buf buf[PD];
#pragma unroll
      for (int k = 0; k < PD - 1; ++k)
        if (k < nu) load(buf[k]);
      for (int ui = 0; ui < nu; ui += PD) {
#pragma unroll
        for (int k = 0; k < PD; ++k) {
          const int uk = ui + k;
          if (uk < nu) {
            if (uk + PD - 1 < nu) load(buf[(k + PD - 1) % PD]);
            compute(buf[k]);
          }
        }
      }
    }
  }
  // the positions past the list up to the next multiple of 16 read as zero
  if (c == G - 1 && tid < kTok * kPosStep) {
    const int t = tid / kPosStep, p = V + tid % kPosStep;
    if (p < ((V + kPosStep - 1) / kPosStep) * kPosStep) {
      a.a_hi[(size_t)t * a.a_stride + p] = __float2half_rn(0.f);
      a.a_lo[(size_t)t * a.a_stride + p] = __float2half_rn(0.f);
    }
  }
  __syncthreads();

  // ================================================================ step 4
  const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * kStages * kStageBytes);
  // a warp's partial of a finished tile goes to its stage that is free at
  // that point (the one consumed last); free_s tells the others where
  __shared__ int free_s[kWarps];
  const char *Wd = reinterpret_cast<const char *>(a.w_down_t);
  int K = 0;
  for (int t = ta; t <= tb; ++t) K += warp_count(t, warp);
  // walks this warp's units in order (k-th unit = (tile t, step s)); one step
  // costs a few integer operations, so the per-unit bookkeeping stays off the
  // path of the copies
  struct Cursor {
    int k, t, s, rem;  // rem: this warp's units of tile t after this one
  };
  auto cursor_tile = [&](Cursor &cu) {  // first unit of the first tile >= cu.t with units
    for (; cu.t <= tb; ++cu.t) {
      const int n = warp_count(cu.t, warp);
      if (n > 0) {
        int sa, sb;
        tile_steps(cu.t, sa, sb);
        cu.s = sa + warp;
        cu.rem = n - 1;
        return;
      }
    }
  };
  auto cursor_next = [&](Cursor &cu) {
    ++cu.k;
    if (cu.rem > 0) {
      cu.s += kWarps;
      --cu.rem;
    } else {
      ++cu.t;
      cursor_tile(cu);
    }
  };
  Cursor fc{0, ta, 0, 0};
  cursor_tile(fc);
  auto issue_acts = [&](int k, int s) {
    const uint32_t st = ring + (uint32_t)((k % kStages) * kStageBytes);
    const int hl = lane >> 4, t8 = (lane >> 1) & 7, half = lane & 1;
    const __half *src = (hl ? a.a_lo : a.a_hi) + (size_t)t8 * a.a_stride + (size_t)s * kPosStep + half * 8;
    cp_async16(st + (uint32_t)(kPosStep * kRowBytes + hl * (kTok * kPosStep * 2) + t8 * 32 + half * 16), src);
  };
  // list ids of the rows this lane copies for the cursor's unit (rows
  // lane / 8 + 4 i), fetched one unit ahead of its copies
  auto fetch_ids = [&](const Cursor &cu, int (&id)[4], bool local) {
    if (cu.k < K) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = (lane >> 3) + 4 * i, p = cu.s * kPosStep + row;
        id[i] = local ? pro_ids_s[warp][cu.k][row] : (p < V ? vid(p) : -1);
      }
    }
  };
  auto issue = [&](int k, int t, int s, const int (&id)[4], bool rows, bool acts) {
    if (k < K) {
      const uint32_t st = ring + (uint32_t)((k % kStages) * kStageBytes);
      if (rows) {
        const char *col = Wd + (size_t)t * kRowBytes + (lane & 7) * 16;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = (lane >> 3) + 4 * i, ch = lane & 7;
          const uint32_t dst = st + (uint32_t)(row * kRowBytes + ((ch ^ (row & 7)) << 4));
          if (id[i] >= 0)
            cp_async16(dst, col + (size_t)id[i] * rb);
          else
            st_shared_zero16(dst);
        }
      }
      if (acts) issue_acts(k, s);
    }
    cp_async_commit();
  };

  // the first stages' weight rows do not depend on step 3: in flight during
  // the grid-wide wait
  int ids_next[4];
  int pro_s[kStages - 1];
#pragma unroll
  for (int k = 0; k < kStages - 1; ++k) {
    fetch_ids(fc, ids_next, true);
    issue(k, fc.t, fc.s, ids_next, true, false);
    pro_s[k] = fc.s;
    cursor_next(fc);
  }
  fetch_ids(fc, ids_next, true);
  int nx_t = fc.t, nx_s = fc.s;  // the unit ids_next belong to (unit kStages - 1)
  cursor_next(fc);
  if (tid == 0) grid_barrier(a.bar, G, c, a.status, a.wait_ns);
  __syncthreads();
  pdl_launch_dependents();
  // their activations, as one more group
#pragma unroll
  for (int k = 0; k < kStages - 1; ++k)
    if (k < K) issue_acts(k, pro_s[k]);
  cp_async_commit();

  if (W == 0) {  // empty list: y = 0
    if (!a.accumulate)
      for (int k = c * kThreads + tid; k < B * d; k += G * kThreads) a.out[k] = 0.f;
    return;
  }

  float acc_h[4][4], acc_l[4][4];
#pragma unroll
  for (int mt = 0; mt < 4; ++mt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc_h[mt][e] = acc_l[mt][e] = 0.f;
  int k = 0;
  for (int t = ta; t <= tb; ++t) {
    const int nt = warp_count(t, warp);
    for (int n = 0; n < nt; ++n, ++k) {
      static_assert(kStages == 3, "the waits below count the groups of a 3-stage ring");
      if (k == 0)
        cp_async_wait<0>();
      else
        cp_async_wait<1>();
      __syncwarp();
      const uint32_t st = ring + (uint32_t)((k % kStages) * kStageBytes);
      const uint32_t ab = st + kPosStep * kRowBytes;
      uint32_t bh0, bh1, bl0, bl1;
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bh0) : "r"(ab + g * 32 + q * 4));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bh1) : "r"(ab + g * 32 + 16 + q * 4));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bl0) : "r"(ab + kTok * kPosStep * 2 + g * 32 + q * 4));
      asm volatile("ld.shared.u32 %0, [%1];" : "=r"(bl1) : "r"(ab + kTok * kPosStep * 2 + g * 32 + 16 + q * 4));
      const int mi = lane >> 3, r = lane & 7, row = r + 8 * (mi >> 1);
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        const int ch = 2 * mt + (mi & 1);
        uint32_t A[4];
        ldmatrix_x4_trans(st + (uint32_t)(row * kRowBytes + ((ch ^ r) << 4)), A);
        mma_16816(acc_h[mt], A, bh0, bh1);
        mma_16816(acc_l[mt], A, bl0, bl1);
      }
      __syncwarp();
      issue(k + kStages - 1, nx_t, nx_s, ids_next, true, true);
      fetch_ids(fc, ids_next, false);
      nx_t = fc.t;
      nx_s = fc.s;
      cursor_next(fc);
    }
    // this warp's partial of tile t, in its free stage (k units consumed:
    // units k .. k + kStages - 2 are in flight, stage (k - 1) mod kStages is free)
    const int fs = (k + kStages - 1) % kStages;
    if (lane == 0) free_s[warp] = fs;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      float *dst = reinterpret_cast<float *>(smem + (size_t)(warp * kStages + fs) * kStageBytes);
      const int col = 16 * mt + g;
      *reinterpret_cast<float2 *>(dst + col * kTok + 2 * q) =
          make_float2(acc_h[mt][0] + acc_l[mt][0], acc_h[mt][1] + acc_l[mt][1]);
      *reinterpret_cast<float2 *>(dst + (col + 8) * kTok + 2 * q) =
          make_float2(acc_h[mt][2] + acc_l[mt][2], acc_h[mt][3] + acc_l[mt][3]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc_h[mt][e] = acc_l[mt][e] = 0.f;
    }
    __syncthreads();
    // tile sum over the warps (in warp order); item = column * 8 + token
    const int col = tid >> 3, tok = tid & 7;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w)
      v += reinterpret_cast<const float *>(smem + (size_t)(w * kStages + free_s[w]) * kStageBytes)[tid];
    const long long tlo = (long long)t * S, thi = tlo + S;
    const int cf = span_owner(W, tlo, G), cl = span_owner(W, thi - 1, G);
    float *y = a.out + (size_t)tok * d + (size_t)t * kTileCols + col;
    if (cf == cl) {
      if (tok < B) *y = a.accumulate ? *y + v : v;
    } else {
      const int slot = (t == ta) ? 0 : 1;
      a.part[((size_t)c * 2 + slot) * kPieceFloats + tid] = v;
      __threadfence();
      __syncthreads();
      if (tid == 0) {
        int pieces = 0;
        for (int cc = cf; cc <= cl; ++cc) pieces += span_lo(W, cc + 1, G) > span_lo(W, cc, G) ? 1 : 0;
        const unsigned old = atomicAdd(&a.ctr[t], 1u);
        last_s = (old == (unsigned)(pieces - 1)) ? 1 : 0;
        if (last_s) {
          a.ctr[t] = 0u;
          __threadfence();
        }
      }
      __syncthreads();
      if (last_s) {
        float s = 0.f;
        for (int cc = cf; cc <= cl; ++cc) {
          const long long clo = span_lo(W, cc, G), chi = span_lo(W, cc + 1, G);
          if (chi <= clo) continue;
          const int sl = (t == (int)(clo / S)) ? 0 : 1;
          s += __ldcg(a.part + ((size_t)cc * 2 + sl) * kPieceFloats + tid);
        }
        if (tok < B) *y = a.accumulate ? *y + s : s;
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
}


// ================================================================ predictor (batches of 2..8)
// One persistent kernel, one CTA per SM, for steps 1-2 of a token batch.  It
// uses the same tensor-core row dot as step 3: weight rows as A fragments
// loaded with 256-bit loads (elements 16q .. 16q + 15 of a 64-element unit
// per lane), the tokens (or h) as the B operand in the matching K order.
//   P1: CTA c computes h for P1 rows 8c .. 8c + 7 (MMA rows 8..15 are zero),
//       K = d split over the 16 warps, partials added in warp order.
//   one grid-wide wait (bounded): h complete.
//   P2: the CTA walks the 32-row words c, c + G, ... (one mask word per
//       token); warp w takes group w & 1 (16 rows) and the eighth w >> 1 of
//       the rank, so its B fragments of h (split into fp16 h_hi and
//       h_lo = fp16(h - h_hi), two MMAs, about 22 bits of h) are built once.
//       The next word's rows are loaded while the current one is reduced.
// Neither P1 nor P2 rows depend on the previous kernel: the CTA's P1 rows and
// its first P2 word are loaded before griddepcontrol.wait, the second word
// before the grid-wide wait, so both are in flight while h is exchanged.
struct PredArgs {
  const __half *p1, *p2;
  const float *p_bias;
  const __half *u;  // [B x d]
  float *h;         // [B x r]
  int d, r, f, B;
  uint32_t *mask;    // [B x nwords]
  uint32_t *uwords;  // [nwords], OR of the tokens' words
  int nwords;
  unsigned *bar;     // grid-barrier word
  int *status;
  unsigned long long wait_ns;
};
constexpr int kPredHRows = 8;   // P1 rows per CTA
constexpr int kPredHUnits = 8;  // P1 64-element units per warp (d <= 8192)
constexpr int kPredSUnits = 2;  // P2 units per warp (2 groups x 8 parts of the rank <= 1024)

PI_DEV uint4 ld_cg16(const void *p) {
  uint4 v;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
PI_DEV float4 ld_cg_f4(const float *p) {
  float4 v;
  asm volatile("ld.global.cg.v4.f32 {%0,%1,%2,%3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

struct PredSBuf {
  uint4 w[kPredSUnits][4];  // [unit][row g lo, row g hi, row g+8 lo, row g+8 hi]
};
__global__ void __launch_bounds__(kThreads, 1) pred_batch_kernel(const __grid_constant__ PredArgs a) {
  __shared__ float red[kWarps][128];
  __shared__ uint32_t uw_s[kTok];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, q = lane & 3;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, r = a.r, f = a.f, nw = a.nwords;

  // ---- P1 rows of this CTA, and its first P2 word, before the wait
  const int j = c * kPredHRows + g;
  const int ns = d / kKStep;
  const int w0 = ns * warp / kWarps, w1 = ns * (warp + 1) / kWarps;
  uint4 wl[kPredHUnits], wh[kPredHUnits];
#pragma unroll
  for (int i = 0; i < kPredHUnits; ++i) {
    wl[i] = wh[i] = make_uint4(0u, 0u, 0u, 0u);
    if (w0 + i < w1 && j < r) ld_stream32(a.p1 + (size_t)j * d + (size_t)(w0 + i) * kKStep + q * 16, wl[i], wh[i]);
  }
  const int grp = warp & 1, part = warp >> 1;
  const int nsr = r / kKStep;
  const int u0 = nsr * part / 8, u1 = nsr * (part + 1) / 8;
  auto load = [&](PredSBuf &b, int word) {
    const int i0 = word * 32 + 16 * grp + g, i1 = i0 + 8;
#pragma unroll
    for (int i = 0; i < kPredSUnits; ++i) {
      b.w[i][0] = b.w[i][1] = b.w[i][2] = b.w[i][3] = make_uint4(0u, 0u, 0u, 0u);
      if (word < nw && u0 + i < u1) {
        const size_t off = (size_t)(u0 + i) * kKStep + q * 16;
        if (i0 < f) ld_stream32(a.p2 + (size_t)i0 * r + off, b.w[i][0], b.w[i][1]);
        if (i1 < f) ld_stream32(a.p2 + (size_t)i1 * r + off, b.w[i][2], b.w[i][3]);
      }
    }
  };
  PredSBuf b0, b1;
  int word = c;
  load(b0, word);
  pdl_wait();

  // ---- P1: h[t][j] = P1_j . u_t
  {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kPredHUnits; ++i) {
      if (w0 + i < w1) {
        uint4 ub0 = make_uint4(0u, 0u, 0u, 0u), ub1 = ub0;
        if (g < a.B) {
          const __half *up = a.u + (size_t)g * d + (size_t)(w0 + i) * kKStep + q * 16;
          ub0 = ld_cg16(up);
          ub1 = ld_cg16(up + 8);
        }
        const uint4 &x0 = wl[i], &x1 = wh[i];
        {
          const uint32_t A[4] = {x0.x, 0u, x0.y, 0u};
          mma_16816(acc, A, ub0.x, ub0.y);
        }
        {
          const uint32_t A[4] = {x0.z, 0u, x0.w, 0u};
          mma_16816(acc, A, ub0.z, ub0.w);
        }
        {
          const uint32_t A[4] = {x1.x, 0u, x1.y, 0u};
          mma_16816(acc, A, ub1.x, ub1.y);
        }
        {
          const uint32_t A[4] = {x1.z, 0u, x1.w, 0u};
          mma_16816(acc, A, ub1.z, ub1.w);
        }
      }
    }
    // lane (g, q) holds row g, tokens 2q and 2q + 1
    red[warp][lane * 2] = acc[0];
    red[warp][lane * 2 + 1] = acc[1];
    __syncthreads();
    if (tid < kPredHRows * kTok) {
      const int row = tid >> 3, t = tid & 7;
      const int jr = c * kPredHRows + row;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += red[w][(row * 4 + (t >> 1)) * 2 + (t & 1)];
      if (t < a.B && jr < r) a.h[(size_t)t * r + jr] = v;
    }
    __syncthreads();
  }
  // the second word's rows stream in during the wait (the P1 registers are free)
  load(b1, word + G);
  // every CTA's slice of h written
  if (tid == 0) grid_barrier(a.bar, G, c, a.status, a.wait_ns);
  __syncthreads();
  pdl_launch_dependents();

  // ---- P2: this warp's h fragments, token g, unit elements 16q .. 16q + 15
  uint32_t hh[kPredSUnits][8], hl[kPredSUnits][8];
#pragma unroll
  for (int i = 0; i < kPredSUnits; ++i)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      hh[i][e] = hl[i][e] = 0u;
    }
#pragma unroll
  for (int i = 0; i < kPredSUnits; ++i) {
    if (g < a.B && u0 + i < u1) {
      const float *hp = a.h + (size_t)g * r + (size_t)(u0 + i) * kKStep + q * 16;
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const float4 x = ld_cg_f4(hp + 4 * v4);
        hh[i][2 * v4] = fused::h_part_pair(x.x, x.y, 0);
        hl[i][2 * v4] = fused::h_part_pair(x.x, x.y, 1);
        hh[i][2 * v4 + 1] = fused::h_part_pair(x.z, x.w, 0);
        hl[i][2 * v4 + 1] = fused::h_part_pair(x.z, x.w, 1);
      }
    }
  }
  auto word_out = [&](const PredSBuf &b, int wd) {
    float acc_h[4] = {0.f, 0.f, 0.f, 0.f}, acc_l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < kPredSUnits; ++i) {
      if (u0 + i < u1) {
        const uint4 &x0 = b.w[i][0], &x1 = b.w[i][1], &y0 = b.w[i][2], &y1 = b.w[i][3];
        const uint32_t A0[4] = {x0.x, y0.x, x0.y, y0.y}, A1[4] = {x0.z, y0.z, x0.w, y0.w};
        const uint32_t A2[4] = {x1.x, y1.x, x1.y, y1.y}, A3[4] = {x1.z, y1.z, x1.w, y1.w};
        mma_16816(acc_h, A0, hh[i][0], hh[i][1]);
        mma_16816(acc_l, A0, hl[i][0], hl[i][1]);
        mma_16816(acc_h, A1, hh[i][2], hh[i][3]);
        mma_16816(acc_l, A1, hl[i][2], hl[i][3]);
        mma_16816(acc_h, A2, hh[i][4], hh[i][5]);
        mma_16816(acc_l, A2, hl[i][4], hl[i][5]);
        mma_16816(acc_h, A3, hh[i][6], hh[i][7]);
        mma_16816(acc_l, A3, hl[i][6], hl[i][7]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) red[warp][lane * 4 + e] = acc_h[e] + acc_l[e];
    __syncthreads();
    // warps 0..7: token t = warp, lane = row of the word (group lane >> 4)
    if (warp < kTok) {
      const int t = warp, row = lane, gr = row >> 4, m = row & 15;
      const int ln = (m & 7) * 4 + (t >> 1), e = (t & 1) + ((m >> 3) << 1);
      const int i = wd * 32 + row;
      float sv = 0.f;
#pragma unroll
      for (int pp = 0; pp < 8; ++pp) sv += red[2 * pp + gr][ln * 4 + e];
      const bool fire = t < a.B && i < f && sv + a.p_bias[i < f ? i : 0] > 0.f;
      const uint32_t bits = __ballot_sync(0xffffffffu, fire);
      if (lane == 0) {
        if (t < a.B) a.mask[(size_t)t * nw + wd] = bits;
        uw_s[t] = bits;
      }
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t u = 0u;
#pragma unroll
      for (int t = 0; t < kTok; ++t) u |= uw_s[t];
      a.uwords[wd] = u;
    }
  };
  for (; word < nw; word += 2 * G) {
    word_out(b0, word);
    load(b0, word + 2 * G);
    if (word + G >= nw) break;
    word_out(b1, word + G);
    load(b1, word + 3 * G);
  }
}

}  // namespace batch
}  // namespace pi
