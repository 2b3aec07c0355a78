// pi_fused.cuh -- one persistent kernel per layer for the batch-1 decode step
// (PowerInfer summary page: Summary, per-layer predictor and neuron-level
// sparse kernels; Interesting ideas I1 hot/cold reordering, I4 kernels that
// read the rows of the active neurons directly).
//
// Grid: one CTA per SM, launched cooperatively (all CTAs co-resident).
// Block: 8 consumer warps + 1 producer warp.  The producer streams work
// items into a ring of 6 x 32 KB shared-memory slots with cp.async.bulk (TMA
// bulk copies) and mbarrier transaction counts; consumers process the slots in
// order:
//   P1 item     rows of P1 owned by this CTA -> its slice of h = P1 u
//               (then a grid-wide barrier publishes all of h)
//   P2 tile     16 predictor rows -> s = P2 h + bias, fire iff s > 0; the
//               tile's active ids go to an in-CTA queue the producer reads
//   GATHER      up (+gate) and down rows of 1-4 active neurons: dot with u,
//               activation, then y += a * W2T_i into per-thread registers
//   DONE        end of the stream
// The producer issues P2 tiles while the consumers wait on the h barrier,
// so the memory system keeps streaming, and issues a tile's gather rows as
// soon as its actives are published.  Tiles of 16 neurons are dealt round
// robin to the CTAs; in dense hot-prefix mode the prefix tiles' rows are
// issued with the tile, without waiting for the predictor.
// After the stream every CTA writes its fp32 partial of y; a second grid
// barrier; each CTA then sums a column slice over all partials in CTA order
// (deterministic, no atomics) and writes y (or adds it to the residual x).
// Every wait is bounded (about 2 s); on expiry the kernel records
// PI_ERR_TIMEOUT in the workspace status word and completes.
#pragma once

#include "pi_device.cuh"

namespace pi {
namespace fused {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kSlots = 6;
constexpr int kSlotBytes = 32768;
constexpr int kTN = 16;          // neurons per predictor tile
constexpr int kMaxGN = 4;        // neurons per gather item
constexpr int kActCap = 2048;    // own active-queue capacity (>= own neurons)
constexpr int kMaxOwnTiles = 128;
constexpr unsigned long long kWaitNs = 2000000000ull;

enum ItemType : int { IT_P1 = 0, IT_P2 = 1, IT_GATHER = 2, IT_DONE = 3 };

struct SlotMeta {
  int type, n, first;
  int ids[kMaxGN];
};

struct Smem {
  uint8_t ring[kSlots][kSlotBytes];
  SlotMeta meta[kSlots];
  unsigned long long full[kSlots];
  unsigned long long empty[kSlots];
  unsigned tbits[kSlots];
  int act[kActCap];
  uint16_t own_bits[kMaxOwnTiles];
  float red[2][kConsumerWarps][2 * kMaxGN];
  double dred[kConsumerWarps];
  float fin[kConsumerWarps][33];
  int iscan[kConsumerWarps];
  volatile int act_tail;
  volatile int tiles_done;
  volatile int abort_flag;
};

struct Args {
  const void *w_up, *w_gate, *w_down_t;
  const __half *s_up, *s_gate, *s_down_t;
  const float *b_up;
  const __half *p1, *p2;
  const float *p_bias;
  const void *in;  // u fp16 [d], or x fp32 [d] in stack mode
  float *out;      // y [d], or x (stack mode, updated in place)
  int d, f, r;
  int stack;       // input is the residual x: RMS-normalise it, and add y into it
  int accumulate;  // y += (non-stack)
  int H;           // dense hot-prefix neurons (multiple of 16); 0 = index mode
  float *h;        // workspace [r]
  float *partial;  // workspace [G x d]
  uint16_t *mask16;  // workspace [ceil(f/16)], written when idx != nullptr
  unsigned *bar;     // workspace grid-barrier word
  int *status;
  int32_t *idx;    // optional ascending active ids [f]
  int32_t *count;  // optional [1]
};

// ---------------------------------------------------------------- PTX helpers
PI_DEV uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
PI_DEV unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
PI_DEV void mbar_init(unsigned long long *b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
PI_DEV void mbar_arrive_tx(unsigned long long *b, unsigned tx) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(tx) : "memory");
}
PI_DEV void mbar_arrive(unsigned long long *b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
PI_DEV bool mbar_try(unsigned long long *b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait; false on timeout (status recorded)
PI_DEV bool mbar_wait(unsigned long long *b, unsigned parity, int *status) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (;;) {
    for (int k = 0; k < 64; ++k)
      if (mbar_try(b, parity)) return true;
    if (globaltimer() - t0 > kWaitNs) {
      set_status(status, kStatusTimeout);
      return false;
    }
  }
}
PI_DEV void bulk_g2s(void *dst, const void *src, unsigned bytes, unsigned long long *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
PI_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
PI_DEV unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
PI_DEV float ld_cg(const float *p) { return __ldcg(p); }

// Grid-wide barrier, one thread per CTA.  Every CTA adds 1 except CTA 0,
// which adds 2^31 - (G - 1): the word's top bit flips exactly when all G
// have arrived, and the low bits return to their previous value, so the
// word never needs resetting between barriers or launches.
PI_DEV bool grid_barrier(unsigned *bar, int G, int c, int *status) {
  const unsigned inc = (c == 0) ? (0x80000000u - (unsigned)(G - 1)) : 1u;
  __threadfence();
  const unsigned old = atomicAdd(bar, inc);
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (((ld_acquire(bar) ^ old) & 0x80000000u) != 0u) return true;
    if (globaltimer() - t0 > kWaitNs) {
      set_status(status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

// ---------------------------------------------------------------- element types
// A consumer thread owns column "chunks": 8 elements (16 B) of fp16 rows or
// 16 elements (8 B) of int4 rows: chunks t, t + 256, t + 512, ...
template <int WT> struct Cols;
template <> struct Cols<W_F16> {
  static constexpr int EC = 8;  // elements per chunk
};
template <> struct Cols<W_INT4> {
  static constexpr int EC = 16;
};

PI_DEV float dot8_h(const uint4 &w, const float *u) {
  float wf[8];
  h8_to_f8(w, wf);
  float a = wf[0] * u[0];
#pragma unroll
  for (int k = 1; k < 8; ++k) a = fmaf(wf[k], u[k], a);
  return a;
}
// 16 int4 values (one 8-byte word pair) times u, without the group scale
PI_DEV float dot16_q(uint2 w, const float *u) {
  float a = 0.f;
  const uint32_t ws[2] = {w.x, w.y};
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int k = 0; k < 8; ++k) a = fmaf((float)((int)((ws[j] >> (4 * k)) & 15u) - 8), u[8 * j + k], a);
  }
  return a;
}

// P1 rows per work item (one slot, at most 4 so that a thread keeps 4 sums)
PI_DEV int p1_rows_per_item(int d) { return min(4, kSlotBytes / (d * 2)); }

// bytes of one weight row and of one int4 scale row
template <int WT>
PI_DEV unsigned wrow_bytes(int d) {
  return WT == W_F16 ? (unsigned)d * 2u : (unsigned)d / 2u;
}
template <int WT>
PI_DEV unsigned srow_bytes(int d) {
  return WT == W_INT4 ? (unsigned)d / 16u : 0u;
}

// Layout of one neuron inside a gather slot: up row, [gate row], down row,
// then (int4) up scales, [gate scales], down scales.
template <int WT, int ACT>
struct NeuronLayout {
  unsigned up, gate, down, sup, sgate, sdown, bytes;
  PI_DEV NeuronLayout(int d) {
    const unsigned rb = wrow_bytes<WT>(d), sb = srow_bytes<WT>(d);
    unsigned o = 0;
    up = o;
    o += rb;
    gate = o;
    if (ACT == ACT_SWIGLU) o += rb;
    down = o;
    o += rb;
    sup = o;
    o += sb;
    sgate = o;
    if (ACT == ACT_SWIGLU) o += sb;
    sdown = o;
    o += sb;
    bytes = o;
  }
};

// ---------------------------------------------------------------- producer
template <int WT, int ACT>
PI_DEV void producer(Smem &S, const Args &a, int c, int G) {
  const int d = a.d, f = a.f, r = a.r;
  const int ntiles = (f + kTN - 1) / kTN;
  const int nown = (c < ntiles) ? (ntiles - 1 - c) / G + 1 : 0;
  const int j0 = (int)((long long)c * r / G), j1 = (int)((long long)(c + 1) * r / G);
  const int rpi = p1_rows_per_item(d);
  const NeuronLayout<WT, ACT> NL(d);
  const int GN = min(kMaxGN, kSlotBytes / (int)NL.bytes);
  const unsigned rb = wrow_bytes<WT>(d), sb = srow_bytes<WT>(d);
  unsigned pn = 0;
  bool ok = true;

  auto acquire = [&](int &s) -> bool {
    s = (int)(pn % kSlots);
    const unsigned par = ((pn / kSlots) & 1u) ^ 1u;
    if (!mbar_wait(&S.empty[s], par, a.status)) {
      S.abort_flag = 1;
      return false;
    }
    return true;
  };
  auto issue_gather = [&](const int *ids, int n) -> bool {
    int s;
    if (!acquire(s)) return false;
    SlotMeta &m = S.meta[s];
    m.type = IT_GATHER;
    m.n = n;
    m.first = 0;
    for (int g = 0; g < n; ++g) m.ids[g] = ids[g];
    mbar_arrive_tx(&S.full[s], NL.bytes * (unsigned)n);
    uint8_t *dst = S.ring[s];
    for (int g = 0; g < n; ++g) {
      const size_t i = (size_t)ids[g];
      uint8_t *nd = dst + g * NL.bytes;
      bulk_g2s(nd + NL.up, (const char *)a.w_up + i * rb, rb, &S.full[s]);
      if (ACT == ACT_SWIGLU) bulk_g2s(nd + NL.gate, (const char *)a.w_gate + i * rb, rb, &S.full[s]);
      bulk_g2s(nd + NL.down, (const char *)a.w_down_t + i * rb, rb, &S.full[s]);
      if (WT == W_INT4) {
        bulk_g2s(nd + NL.sup, (const char *)a.s_up + i * sb, sb, &S.full[s]);
        if (ACT == ACT_SWIGLU) bulk_g2s(nd + NL.sgate, (const char *)a.s_gate + i * sb, sb, &S.full[s]);
        bulk_g2s(nd + NL.sdown, (const char *)a.s_down_t + i * sb, sb, &S.full[s]);
      }
    }
    ++pn;
    return true;
  };

  // 1. this CTA's rows of P1
  for (int j = j0; ok && j < j1; j += rpi) {
    const int n = min(rpi, j1 - j);
    int s;
    if (!(ok = acquire(s))) break;
    S.meta[s].type = IT_P1;
    S.meta[s].n = n;
    S.meta[s].first = j;
    const unsigned bytes = (unsigned)n * (unsigned)d * 2u;
    mbar_arrive_tx(&S.full[s], bytes);
    bulk_g2s(S.ring[s], a.p1 + (size_t)j * d, bytes, &S.full[s]);
    ++pn;
  }
  // 2. predictor tiles and gather rows
  int k = 0, taken = 0;
  unsigned long long t0 = 0;
  while (ok) {
    const int tail = S.act_tail;
    __threadfence_block();
    if (taken < tail) {
      const int n = min(GN, tail - taken);
      ok = issue_gather(&S.act[taken], n);
      taken += n;
      t0 = 0;
      continue;
    }
    if (k < nown) {
      const int tile = c + k * G;
      const int rows = min(kTN, f - tile * kTN);
      int s;
      if (!(ok = acquire(s))) break;
      S.meta[s].type = IT_P2;
      S.meta[s].n = rows;
      S.meta[s].first = tile;
      S.tbits[s] = 0u;
      const unsigned bytes = (unsigned)rows * (unsigned)r * 2u;
      mbar_arrive_tx(&S.full[s], bytes);
      bulk_g2s(S.ring[s], a.p2 + (size_t)tile * kTN * r, bytes, &S.full[s]);
      ++pn;
      if (tile * kTN < a.H) {  // dense hot prefix: every row of the tile, now
        int ids[kMaxGN];
        for (int q = 0; ok && q < rows; q += GN) {
          const int n = min(GN, rows - q);
          for (int g = 0; g < n; ++g) ids[g] = tile * kTN + q + g;
          ok = issue_gather(ids, n);
        }
      }
      ++k;
      t0 = 0;
      continue;
    }
    if (S.tiles_done == nown) {
      __threadfence_block();
      if (S.act_tail == taken) break;
      continue;
    }
    if (S.abort_flag) {
      ok = false;
      break;
    }
    if (t0 == 0) t0 = globaltimer();
    if (globaltimer() - t0 > kWaitNs) {
      set_status(a.status, kStatusTimeout);
      S.abort_flag = 1;
      ok = false;
      break;
    }
    __nanosleep(32);
  }
  // 3. end of stream (also after an abort, so consumers stop)
  int s;
  if (acquire(s)) {
    S.meta[s].type = IT_DONE;
    S.meta[s].n = 0;
    mbar_arrive(&S.full[s]);
  } else {
    S.abort_flag = 1;
  }
}

// ---------------------------------------------------------------- kernel
// CPT: column chunks per consumer thread (d <= CPT * 256 * EC)
template <int WT, int ACT, int CPT>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem &S = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  constexpr int EC = Cols<WT>::EC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, f = a.f, r = a.r;

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kConsumerWarps);
    }
    S.act_tail = 0;
    S.tiles_done = 0;
    S.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (warp == kConsumerWarps) {
    if (lane == 0) producer<WT, ACT>(S, a, c, G);
    return;
  }

  // ------------------------------------------------------------ consumers
  const int nch = d / EC;
  const int ntiles = (f + kTN - 1) / kTN;
  const int j0 = (int)((long long)c * r / G), j1 = (int)((long long)(c + 1) * r / G);
  const int rpi = p1_rows_per_item(d);
  const int n_p1 = (j1 - j0 + rpi - 1) / rpi;
  const NeuronLayout<WT, ACT> NL(d);

  // FFN input u for the owned columns (fp32 registers)
  float u[CPT][EC];
  if (a.stack) {
    const float *x = reinterpret_cast<const float *>(a.in);
    double ss = 0.0;
    for (int k = tid; k < d; k += kConsumers) {
      const double v = (double)x[k];
      ss += v * v;
    }
    ss = warp_sum_d(ss);
    if (lane == 0) S.dred[warp] = ss;
    consumer_sync();
    double tot = 0.0;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) tot += S.dred[w];
    const float mean = __double2float_rn(tot / (double)d);
    const float den = __fsqrt_rn(__fadd_rn(mean, 1e-6f));
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int ch = tid + q * kConsumers;
#pragma unroll
      for (int e = 0; e < EC; ++e)
        u[q][e] = (ch < nch) ? __half2float(__float2half_rn(__fdiv_rn(x[ch * EC + e], den))) : 0.f;
    }
  } else {
    const __half *uh = reinterpret_cast<const __half *>(a.in);
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const int ch = tid + q * kConsumers;
#pragma unroll
      for (int e = 0; e < EC; e += 8) {
        if (ch < nch) {
          h8_to_f8(ld_keep16(uh + ch * EC + e), &u[q][e]);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) u[q][e + k] = 0.f;
        }
      }
    }
  }
  float y[CPT][EC];
#pragma unroll
  for (int q = 0; q < CPT; ++q)
#pragma unroll
    for (int e = 0; e < EC; ++e) y[q][e] = 0.f;

  unsigned n = 0;   // items consumed
  unsigned nr = 0;  // reductions done (parity of the red buffer)
  bool alive = true;
  auto wait_full = [&](int &s) -> bool {
    s = (int)(n % kSlots);
    if (!mbar_wait(&S.full[s], (n / kSlots) & 1u, a.status)) {
      S.abort_flag = 1;
      return false;
    }
    return true;
  };
  auto release = [&](int s) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[s]);
    ++n;
  };

  // ---- P1 items: this CTA's slice of h
  for (int it = 0; it < n_p1 && alive; ++it) {
    int s;
    if (!(alive = wait_full(s))) break;
    const int rows = S.meta[s].n, jf = S.meta[s].first;
    float part[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) part[q] = 0.f;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (q >= rows) break;
      const __half *row = reinterpret_cast<const __half *>(S.ring[s]) + (size_t)q * d;
      float acc = 0.f;
#pragma unroll
      for (int cq = 0; cq < CPT; ++cq) {
        const int ch = tid + cq * kConsumers;
        if (ch < nch) {
#pragma unroll
          for (int e = 0; e < EC; e += 8)
            acc += dot8_h(*reinterpret_cast<const uint4 *>(row + ch * EC + e), &u[cq][e]);
        }
      }
      part[q] = acc;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) part[q] = warp_sum(part[q]);
    const int par = nr & 1;
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < 4; ++q) S.red[par][warp][q] = part[q];
    }
    release(s);
    consumer_sync();
    ++nr;
    if (tid < rows && tid < 4) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) t += S.red[par][w][tid];
      a.h[jf + tid] = t;
    }
  }
  // ---- h is complete once every CTA got here
  consumer_sync();
  if (tid == 0) {
    if (!grid_barrier(a.bar, G, c, a.status)) S.abort_flag = 1;
  }
  consumer_sync();
  // predictor columns of this lane: chunks lane + 32 kk (8 fp16 each)
  const int pch = r / 8;
  float hreg[4][8];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int ch = lane + 32 * kk;
#pragma unroll
    for (int e = 0; e < 8; ++e) hreg[kk][e] = (ch < pch) ? ld_cg(a.h + ch * 8 + e) : 0.f;
  }

  // ---- main stream
  while (alive) {
    int s;
    if (!(alive = wait_full(s))) break;
    const int type = S.meta[s].type;
    if (type == IT_DONE) {
      release(s);
      break;
    }
    if (type == IT_P2) {
      const int tile = S.meta[s].first, rows = S.meta[s].n;
#pragma unroll
      for (int rr = 0; rr < kTN / kConsumerWarps; ++rr) {
        const int row_i = warp + rr * kConsumerWarps;
        if (row_i < rows) {
          const __half *row = reinterpret_cast<const __half *>(S.ring[s]) + (size_t)row_i * r;
          float acc = 0.f;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const int ch = lane + 32 * kk;
            if (ch < pch) acc += dot8_h(*reinterpret_cast<const uint4 *>(row + ch * 8), hreg[kk]);
          }
          acc = warp_sum(acc);
          const int i = tile * kTN + row_i;
          if (lane == 0 && acc + __ldg(a.p_bias + i) > 0.f) atomicOr(&S.tbits[s], 1u << row_i);
        }
      }
      consumer_sync();
      if (tid == 0) {
        const unsigned bits = S.tbits[s];
        S.own_bits[(tile - c) / G] = (uint16_t)bits;
        if (a.idx || a.count) a.mask16[tile] = (uint16_t)bits;
        if (tile * kTN >= a.H) {
          int t = S.act_tail;
          unsigned b = bits;
          while (b) {
            const int bit = __ffs(b) - 1;
            b &= b - 1u;
            S.act[t++] = tile * kTN + bit;
          }
          __threadfence_block();
          S.act_tail = t;
        }
        __threadfence_block();
        S.tiles_done = S.tiles_done + 1;
      }
      release(s);
      continue;
    }
    // IT_GATHER
    const int ng = S.meta[s].n;
    float part[kMaxGN][2];
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) part[g][0] = part[g][1] = 0.f;
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) {
      if (g < ng) {
        const uint8_t *nd = S.ring[s] + g * NL.bytes;
#pragma unroll
        for (int cq = 0; cq < CPT; ++cq) {
          const int ch = tid + cq * kConsumers;
          if (ch < nch) {
            if (WT == W_F16) {
              part[g][0] += dot8_h(*reinterpret_cast<const uint4 *>(nd + NL.up + ch * 16), u[cq]);
              if (ACT == ACT_SWIGLU)
                part[g][1] += dot8_h(*reinterpret_cast<const uint4 *>(nd + NL.gate + ch * 16), u[cq]);
            } else {
              const float su = __half2float(*reinterpret_cast<const __half *>(nd + NL.sup + (ch >> 1) * 2));
              part[g][0] = fmaf(su, dot16_q(*reinterpret_cast<const uint2 *>(nd + NL.up + ch * 8), u[cq]), part[g][0]);
              if (ACT == ACT_SWIGLU) {
                const float sg = __half2float(*reinterpret_cast<const __half *>(nd + NL.sgate + (ch >> 1) * 2));
                part[g][1] =
                    fmaf(sg, dot16_q(*reinterpret_cast<const uint2 *>(nd + NL.gate + ch * 8), u[cq]), part[g][1]);
              }
            }
          }
        }
      }
    }
    const int par = nr & 1;
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) {
      if (g < ng) {
        const float v0 = warp_sum(part[g][0]);
        const float v1 = (ACT == ACT_SWIGLU) ? warp_sum(part[g][1]) : 0.f;
        if (lane == 0) {
          S.red[par][warp][2 * g] = v0;
          S.red[par][warp][2 * g + 1] = v1;
        }
      }
    }
    consumer_sync();
    ++nr;
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) {
      if (g < ng) {
        float up = 0.f, gt = 0.f;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) {
          up += S.red[par][w][2 * g];
          gt += S.red[par][w][2 * g + 1];
        }
        const int i = S.meta[s].ids[g];
        const int tile = i / kTN;
        const bool member = (S.own_bits[(tile - c) / G] >> (i % kTN)) & 1u;
        float av;
        if (ACT == ACT_RELU)
          av = member ? fmaxf(up + __ldg(a.b_up + i), 0.f) : 0.f;
        else
          av = member ? silu(gt) * up : 0.f;
        if (av != 0.f) {
          const uint8_t *nd = S.ring[s] + g * NL.bytes;
#pragma unroll
          for (int cq = 0; cq < CPT; ++cq) {
            const int ch = tid + cq * kConsumers;
            if (ch < nch) {
              if (WT == W_F16) {
                float w[8];
                h8_to_f8(*reinterpret_cast<const uint4 *>(nd + NL.down + ch * 16), w);
#pragma unroll
                for (int e = 0; e < 8; ++e) y[cq][e] = fmaf(av, w[e], y[cq][e]);
              } else {
                const float sd = __half2float(*reinterpret_cast<const __half *>(nd + NL.sdown + (ch >> 1) * 2));
                const uint2 wq = *reinterpret_cast<const uint2 *>(nd + NL.down + ch * 8);
                const uint32_t ws[2] = {wq.x, wq.y};
                const float as = av * sd;
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                  for (int e = 0; e < 8; ++e)
                    y[cq][8 * j + e] = fmaf(as, (float)((int)((ws[j] >> (4 * e)) & 15u) - 8), y[cq][8 * j + e]);
              }
            }
          }
        }
      }
    }
    release(s);
  }

  if (S.abort_flag && tid == 0) {
    // a wait gave up: let any bulk copy still in flight into this CTA's
    // shared memory land before the CTA can exit (bounded, about 1 ms)
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) __nanosleep(1000);
  }
  // ---- partial of y
#pragma unroll
  for (int cq = 0; cq < CPT; ++cq) {
    const int ch = tid + cq * kConsumers;
    if (ch < nch) {
      float4 *dst = reinterpret_cast<float4 *>(a.partial + (size_t)c * d + (size_t)ch * EC);
#pragma unroll
      for (int e = 0; e < EC; e += 4) dst[e / 4] = make_float4(y[cq][e], y[cq][e + 1], y[cq][e + 2], y[cq][e + 3]);
    }
  }
  consumer_sync();
  if (tid == 0) {
    if (!grid_barrier(a.bar, G, c, a.status)) S.abort_flag = 1;
  }
  consumer_sync();

  // ---- column slice: sum of the G partials in CTA order
  const int cw = (d + G - 1) / G;
  const int c0 = min(d, c * cw), c1 = min(d, c0 + cw);
  const int col_l = tid & 31, grp = tid >> 5;
  for (int base = c0; base < c1; base += 32) {
    const int col = base + col_l;
    float sum = 0.f;
    if (col < c1)
      for (int cc = grp; cc < G; cc += kConsumerWarps) sum += ld_cg(a.partial + (size_t)cc * d + col);
    S.fin[grp][col_l] = sum;
    consumer_sync();
    if (grp == 0 && col < c1) {
      float t = S.fin[0][col_l];
#pragma unroll
      for (int g = 1; g < kConsumerWarps; ++g) t += S.fin[g][col_l];
      a.out[col] = (a.stack || a.accumulate) ? a.out[col] + t : t;
    }
    consumer_sync();
  }

  // ---- ascending active ids (optional): CTA c writes the ids of tiles
  // [c * tpc, (c + 1) * tpc) after the popcount of all earlier tiles
  if (a.idx != nullptr || a.count != nullptr) {
    const int tpc = (ntiles + G - 1) / G;
    const int t0 = min(ntiles, c * tpc), t1 = min(ntiles, t0 + tpc);
    int before = 0;
    for (int t = tid; t < t0; t += kConsumers) before += __popc((unsigned)__ldcg(a.mask16 + t));
    int total = before;
    for (int t = t0 + tid; t < ntiles; t += kConsumers) total += __popc((unsigned)__ldcg(a.mask16 + t));
    before = __reduce_add_sync(0xffffffffu, before);
    total = __reduce_add_sync(0xffffffffu, total);
    if (lane == 0) S.iscan[warp] = before;
    consumer_sync();
    if (tid == 0) {
      int b = 0;
      for (int w = 0; w < kConsumerWarps; ++w) b += S.iscan[w];
      S.iscan[0] = b;
    }
    consumer_sync();
    before = S.iscan[0];
    consumer_sync();
    if (lane == 0) S.iscan[warp] = total;
    consumer_sync();
    if (tid == 0) {
      int tt = 0;
      for (int w = 0; w < kConsumerWarps; ++w) tt += S.iscan[w];
      if (c == 0 && a.count) a.count[0] = tt;
      if (a.idx) {
        int pos = before;
        for (int t = t0; t < t1; ++t) {
          unsigned b = (unsigned)__ldcg(a.mask16 + t);
          while (b) {
            const int bit = __ffs(b) - 1;
            b &= b - 1u;
            a.idx[pos++] = t * kTN + bit;
          }
        }
      }
    }
  }
}

}  // namespace fused
}  // namespace pi
