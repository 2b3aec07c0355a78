// pi_fused.cuh -- one persistent kernel per layer for the batch-1 decode step
// (PowerInfer summary page: Summary, per-layer predictor and neuron-level
// sparse kernels; Interesting ideas I1 hot/cold reordering, I4 kernels that
// read the rows of the active neurons directly).
//
// Grid: one CTA per SM, launched cooperatively (all CTAs co-resident).
// Block: 8 consumer warps + 1 producer warp.  The producer streams work items
// into a ring of 3 x 64 KB shared-memory slots with cp.async.bulk (TMA bulk
// copies) and mbarrier transaction counts; consumers process the slots in
// order:
//   P1 item     up to 8 rows of P1 owned by this CTA -> its slice of h = P1 u
//               (then a grid-wide barrier publishes all of h)
//   P2 tile     32 predictor rows -> s = P2 h + bias, fire iff s > 0.  Warps
//               record the fired bits with shared-memory atomics and release
//               the slot without a block barrier.
//   GATHER      up (+gate) and down rows of 1-4 neurons: dot with u,
//               activation, then y += a * W2T_i in per-thread registers
//   DONE        end of the stream
// The producer "harvests" a tile when its slot's empty barrier completes
// (every consumer warp is done with it), appends the fired ids to its list
// and issues their gather rows; it keeps issuing P2 tiles meanwhile, and it
// prefetches tiles while the consumers wait on the h barrier.  Neurons are
// dealt round robin to the CTAs (neuron i to CTA i mod G), so every CTA gets
// the same mix of hot and cold neurons; CTA c's k-th tile holds its own
// neurons c + (32k + q) G, q < 32.  In dense hot-prefix mode the rows of a
// tile's prefix neurons are issued right after the tile, without waiting
// for its bits.
// After the stream every CTA writes its fp32 partial of y; a second grid
// barrier; each CTA then sums a column slice over all partials in CTA order
// (deterministic, no atomics) and writes y (or adds it to the residual x).
// Every wait is bounded (about 2 s); on expiry the kernel records
// PI_ERR_TIMEOUT in the workspace status word and completes.
#pragma once

#include <cstddef>

#include "pi_device.cuh"

namespace pi {
namespace fused {

constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kSlots = 3;
constexpr int kSlotBytes = 65536;
constexpr int kTN = 32;                      // neurons per predictor tile
constexpr int kMaxGN = 4;                    // neurons per gather item
constexpr int kMaxOwnTiles = 32;             // neurons per CTA <= 32 * 32
constexpr int kActCap = kMaxOwnTiles * kTN;  // capacity of the active-id list
constexpr int kMaxR = 1024;                  // predictor rank
constexpr int kMaxP1Rows = 8;                // P1 rows per item
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
  unsigned tbits[kSlots];              // fired bits of the tile in a slot
  unsigned own_bits[kMaxOwnTiles];     // fired bits of this CTA's tiles
  int act[kActCap];                    // fired ids (index mode), producer-owned
  int tile_item[kMaxOwnTiles];         // item number each own tile was issued as
  float own_pbias[kMaxOwnTiles][kTN];  // predictor bias of this CTA's neurons
  float own_bup[kMaxOwnTiles][kTN];    // ReLU bias b1 of this CTA's neurons
  alignas(16) float h_s[kMaxR];  // written with 16-byte vector stores
  float red[2][kConsumerWarps][2 * kMaxGN];
  double dred[kConsumerWarps];
  float fin[kConsumerWarps][33];
  int iscan[kConsumerWarps];
  volatile int abort_flag;
};

static_assert(offsetof(Smem, ring) == 0, "ring slots must start the shared block");
static_assert(kSlotBytes % 16 == 0, "bulk copies need 16-byte aligned slots");
static_assert(offsetof(Smem, h_s) % 16 == 0, "h_s is accessed with 16-byte vectors");
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory per block");

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
  int H;           // dense hot-prefix neurons [0, H); 0 = index mode
  float *h;        // workspace [r]
  float *partial;  // workspace [G x d]
  unsigned *mask32;  // workspace [ceil(f/32)] fired bits of neurons 32w..32w+31, when idx or count != nullptr
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
// try_wait with a suspend-time hint: the thread is parked until the phase
// completes or the hint (ns) elapses, instead of spinning on the barrier
PI_DEV bool mbar_try(unsigned long long *b, unsigned parity, unsigned hint_ns) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
PI_DEV bool mbar_test(unsigned long long *b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait; false on timeout (status recorded).  The fast path (phase
// already complete) is inline, the suspending loop is out of line to keep
// the consumer loop small in the instruction cache.
__device__ __noinline__ bool mbar_wait_slow(unsigned long long *b, unsigned parity, int *status) {
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_try(b, parity, 20000u)) return true;
    if (globaltimer() - t0 > kWaitNs) {
      set_status(status, kStatusTimeout);
      return false;
    }
  }
}
PI_DEV bool mbar_wait(unsigned long long *b, unsigned parity, int *status) {
  if (mbar_test(b, parity)) return true;
  return mbar_wait_slow(b, parity, status);
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

// dot of 8 fp16 weights with 8 fp32 values as two independent chains
PI_DEV float dot8_h2(const uint4 &w, const float *u) {
  const __half2 *hp = reinterpret_cast<const __half2 *>(&w);
  const float2 a0 = __half22float2(hp[0]), a1 = __half22float2(hp[1]);
  const float2 a2 = __half22float2(hp[2]), a3 = __half22float2(hp[3]);
  float x = a0.x * u[0], y = a0.y * u[1];
  x = fmaf(a1.x, u[2], x);
  y = fmaf(a1.y, u[3], y);
  x = fmaf(a2.x, u[4], x);
  y = fmaf(a2.y, u[5], y);
  x = fmaf(a3.x, u[6], x);
  y = fmaf(a3.y, u[7], y);
  return x + y;
}
// 16 int4 values (one 8-byte word pair) times u, without the group scale,
// as two independent chains
PI_DEV float dot16_q(uint2 w, const float *u) {
  float x = 0.f, y = 0.f;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    x = fmaf((float)((int)((w.x >> (4 * k)) & 15u) - 8), u[k], x);
    y = fmaf((float)((int)((w.y >> (4 * k)) & 15u) - 8), u[8 + k], y);
  }
  return x + y;
}

// 8 fp16 weights times 8 fp16 inputs (16 B each), accumulated into two fp32
// chains with the mixed-precision FMA: the product of two fp16 values is exact
// in fp32, so each step equals fmaf((float)w, (float)u, acc) bit for bit
PI_DEV void dot8_mixed(const uint4 &w, const uint4 &u, float &x, float &y) {
  const unsigned ws[4] = {w.x, w.y, w.z, w.w}, us[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int k = 0; k < 4; ++k)
    asm("{\n .reg .b16 al, ah, bl, bh;\n mov.b32 {al, ah}, %2;\n mov.b32 {bl, bh}, %3;\n"
        " fma.rn.f32.f16 %0, al, bl, %0;\n fma.rn.f32.f16 %1, ah, bh, %1;\n}\n"
        : "+f"(x), "+f"(y)
        : "r"(ws[k]), "r"(us[k]));
}
// the 8 int4 codes of one 32-bit word (element 2k = low nibble of byte k) as
// four fp16 pairs (q - 8): 0x6400 | q is the fp16 value 1024 + q, and
// subtracting 1032 is exact
PI_DEV void q8_to_h2(uint32_t w, uint32_t out[4]) {
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t t = w >> (8 * k);
    const uint32_t hb = (t & 0xFu) | ((t & 0xF0u) << 12) | 0x64006400u;
    const __half2 v = __hsub2(*reinterpret_cast<const __half2 *>(&hb), off);
    out[k] = *reinterpret_cast<const uint32_t *>(&v);
  }
}
// 16 int4 codes (q - 8) times 16 fp16 inputs, without the group scale
PI_DEV void dot16_q_mixed(const uint2 &w, const uint4 &u0, const uint4 &u1, float &x, float &y) {
  uint32_t q[8];
  q8_to_h2(w.x, q);
  q8_to_h2(w.y, q + 4);
  dot8_mixed(make_uint4(q[0], q[1], q[2], q[3]), u0, x, y);
  dot8_mixed(make_uint4(q[4], q[5], q[6], q[7]), u1, x, y);
}

// the 8 int4 codes n0..n7 of one 32-bit word as the fp16 pairs (1024 + n_j,
// 1024 + n_(j+4)), j = 0..3: one shift and one masked OR per pair (0x6400 | q
// is the fp16 value 1024 + q)
PI_DEV uint4 q8_pairs_biased(uint32_t w) {
  return make_uint4((w & 0x000F000Fu) | 0x64006400u, ((w >> 4) & 0x000F000Fu) | 0x64006400u,
                    ((w >> 8) & 0x000F000Fu) | 0x64006400u, ((w >> 12) & 0x000F000Fu) | 0x64006400u);
}
// fp16 pairs (k, k+4) of each 8-element block of 8 fp16 inputs (16 B)
PI_DEV uint4 pair_k4(const uint4 &v) {
  return make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632), __byte_perm(v.y, v.w, 0x5410),
                    __byte_perm(v.y, v.w, 0x7632));
}

// sum N independent values across the warp; the N butterflies are
// interleaved so that their shuffles overlap
template <int N>
PI_DEV void warp_sum_n(float (&v)[N]) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
    for (int k = 0; k < N; ++k) v[k] += __shfl_xor_sync(0xffffffffu, v[k], o);
  }
}

PI_DEV int p1_rows_per_item(int d) { return min(kMaxP1Rows, kSlotBytes / (d * 2)); }

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

// neurons of CTA c: i = c + m G, m < own_count; tile k holds m in [32k, 32k + 32)
PI_DEV int own_count(int f, int c, int G) { return c < f ? (f - 1 - c) / G + 1 : 0; }

// ---------------------------------------------------------------- producer
// The whole producer warp runs this loop in lockstep with identical state;
// lane 0 writes the slot descriptors and arms the mbarriers, and the bulk
// copies of an item are spread over the lanes (one row per lane), so a tile
// of 32 strided rows costs one warp instruction.
template <int WT, int ACT>
PI_DEV void producer(Smem &S, const Args &a, int c, int G, int lane) {
  const int d = a.d, f = a.f, r = a.r;
  const int nn = own_count(f, c, G);
  const int nown = (nn + kTN - 1) / kTN;
  const int j0 = (int)((long long)c * r / G), j1 = (int)((long long)(c + 1) * r / G);
  const int rpi = p1_rows_per_item(d);
  const NeuronLayout<WT, ACT> NL(d);
  const int GN = min(kMaxGN, kSlotBytes / (int)NL.bytes);
  const unsigned rb = wrow_bytes<WT>(d), sb = srow_bytes<WT>(d);
  constexpr int CPN = (ACT == ACT_SWIGLU ? 3 : 2) * (WT == W_INT4 ? 2 : 1);  // copies per neuron
  const bool want_mask = a.idx != nullptr || a.count != nullptr;
  unsigned pn = 0;   // items issued
  int k = 0;         // own tiles issued
  int hk = 0;        // own tiles harvested
  int act_tail = 0;  // fired own indices appended (index mode)
  int taken = 0;     // fired own indices issued as gather items
  bool ok = true;

  // fired bits of own tile hk are final once its slot's empty phase completed
  auto harvest = [&]() {
    const int s = S.tile_item[hk] % kSlots;
    const unsigned bits = S.tbits[s];
    const int fired = __popc(bits);
    if (lane == 0) {
      unsigned b = bits;
      int t = act_tail;
      while (b) {
        const int q = __ffs(b) - 1;
        b &= b - 1u;
        const int m = hk * kTN + q;
        const int i = c + m * G;
        if (want_mask) atomicOr(a.mask32 + (i >> 5), 1u << (i & 31));
        if (i >= a.H) S.act[t++] = m;
      }
    }
    // prefix neurons were issued densely: count only the others (ids grow with q)
    int added = 0;
    unsigned b = bits;
    while (b) {
      const int q = __ffs(b) - 1;
      b &= b - 1u;
      added += (c + (hk * kTN + q) * G >= a.H) ? 1 : 0;
    }
    (void)fired;
    act_tail += added;
    ++hk;
    __syncwarp();
  };
  auto tile_done = [&](int kk) -> bool {
    const unsigned it = (unsigned)S.tile_item[kk];
    return mbar_test(&S.empty[it % kSlots], (it / kSlots) & 1u);
  };
  // next slot in ring order; every tile that lived in a slot freed so far is
  // harvested before its slot is overwritten
  auto acquire = [&](int &s) -> bool {
    s = (int)(pn % kSlots);
    const unsigned par = ((pn / kSlots) & 1u) ^ 1u;
    if (!mbar_wait(&S.empty[s], par, a.status)) {
      if (lane == 0) S.abort_flag = 1;
      return false;
    }
    while (hk < k && (unsigned)S.tile_item[hk] + kSlots <= pn) harvest();
    return true;
  };
  // gather item: own indices ms[0..n); lane j issues copy j
  auto issue_gather = [&](const int *ms, int n) -> bool {
    int s;
    if (!acquire(s)) return false;
    if (lane == 0) {
      SlotMeta &m = S.meta[s];
      m.type = IT_GATHER;
      m.n = n;
      m.first = 0;
      for (int g = 0; g < n; ++g) m.ids[g] = ms[g];
      mbar_arrive_tx(&S.full[s], NL.bytes * (unsigned)n);
    }
    __syncwarp();
    if (lane < n * CPN) {
      const int g = lane / CPN, kind = lane % CPN;
      const size_t i = (size_t)(c + ms[g] * G);
      uint8_t *nd = S.ring[s] + g * NL.bytes;
      const void *src;
      unsigned off, bytes = rb;
      if (kind == 0) {
        src = (const char *)a.w_up + i * rb;
        off = NL.up;
      } else if (ACT == ACT_SWIGLU && kind == 1) {
        src = (const char *)a.w_gate + i * rb;
        off = NL.gate;
      } else if (kind == (ACT == ACT_SWIGLU ? 2 : 1)) {
        src = (const char *)a.w_down_t + i * rb;
        off = NL.down;
      } else {  // int4 scale rows, in the order up, [gate,] down
        const int sk = kind - (ACT == ACT_SWIGLU ? 3 : 2);
        bytes = sb;
        if (sk == 0) {
          src = (const char *)a.s_up + i * sb;
          off = NL.sup;
        } else if (ACT == ACT_SWIGLU && sk == 1) {
          src = (const char *)a.s_gate + i * sb;
          off = NL.sgate;
        } else {
          src = (const char *)a.s_down_t + i * sb;
          off = NL.sdown;
        }
      }
      bulk_g2s(nd + off, src, bytes, &S.full[s]);
    }
    ++pn;
    return true;
  };

  // 1. this CTA's rows of P1
  for (int j = j0; ok && j < j1; j += rpi) {
    const int n = min(rpi, j1 - j);
    int s;
    if (!(ok = acquire(s))) break;
    if (lane == 0) {
      S.meta[s].type = IT_P1;
      S.meta[s].n = n;
      S.meta[s].first = j;
      const unsigned bytes = (unsigned)n * (unsigned)d * 2u;
      mbar_arrive_tx(&S.full[s], bytes);
      bulk_g2s(S.ring[s], a.p1 + (size_t)j * d, bytes, &S.full[s]);
    }
    ++pn;
  }
  // 2. predictor tiles and gather rows
  while (ok) {
    while (hk < k && tile_done(hk)) harvest();
    if (taken < act_tail) {
      const int n = min(GN, act_tail - taken);
      ok = issue_gather(&S.act[taken], n);
      taken += n;
      continue;
    }
    if (k < nown) {
      const int rows = min(kTN, nn - k * kTN);
      int s;
      if (!(ok = acquire(s))) break;
      const unsigned rbp = (unsigned)r * 2u;
      if (lane == 0) {
        S.meta[s].type = IT_P2;
        S.meta[s].n = rows;
        S.meta[s].first = k;
        S.tbits[s] = 0u;
        S.tile_item[k] = (int)pn;
        mbar_arrive_tx(&S.full[s], (unsigned)rows * rbp);
      }
      __syncwarp();
      if (lane < rows) bulk_g2s(S.ring[s] + lane * rbp, a.p2 + (size_t)(c + (k * kTN + lane) * G) * r, rbp, &S.full[s]);
      ++pn;
      // dense hot prefix: the tile's prefix neurons (the smallest ids), now
      int ms[kMaxGN], ng = 0;
      for (int q = 0; ok && q < rows; ++q) {
        if (c + (k * kTN + q) * G >= a.H) break;
        ms[ng++] = k * kTN + q;
        if (ng == GN) {
          ok = issue_gather(ms, ng);
          ng = 0;
        }
      }
      if (ok && ng) ok = issue_gather(ms, ng);
      ++k;
      continue;
    }
    if (hk == nown) break;  // every tile harvested and every fired id issued
    // wait for the consumers to finish the oldest unharvested tile
    const unsigned it = (unsigned)S.tile_item[hk];
    if (!mbar_wait(&S.empty[it % kSlots], (it / kSlots) & 1u, a.status)) {
      if (lane == 0) S.abort_flag = 1;
      ok = false;
      break;
    }
    harvest();
  }
  // 3. end of stream (also after an abort, so consumers stop)
  __threadfence();  // mask words visible before the consumers' grid barrier
  int s;
  if (acquire(s)) {
    if (lane == 0) {
      S.meta[s].type = IT_DONE;
      S.meta[s].n = 0;
      mbar_arrive(&S.full[s]);
    }
  } else if (lane == 0) {
    S.abort_flag = 1;
  }
}

// ---------------------------------------------------------------- kernel
// CPT: column chunks per consumer thread (d <= CPT * 256 * EC)
template <int WT, int ACT, int CPT>
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(Args a) {
  // indexed directly (no integer round trip) so that every access stays in
  // the shared state space; bulk copies need only 16-byte alignment
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem &S = *reinterpret_cast<Smem *>(smem_raw);
  constexpr int EC = Cols<WT>::EC;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const int d = a.d, f = a.f, r = a.r;
  const int nwords = (f + 31) / 32;
  const int nn = own_count(f, c, G);

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kConsumerWarps);
    }
    S.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int k = tid; k < kMaxOwnTiles; k += blockDim.x) S.own_bits[k] = 0u;
  __syncthreads();

  // Programmatic dependent launch: the next step's grid may be scheduled
  // now, and its CTAs take SMs as this grid's CTAs leave.  The producer
  // streams weights only (P1 rows, P2 tiles, weight rows), which no earlier
  // kernel writes, so it starts at once; the consumers wait for the
  // preceding grid before reading the input or touching the workspace.
  pdl_launch_dependents();
  if (warp == kConsumerWarps) {
    producer<WT, ACT>(S, a, c, G, lane);
    return;
  }
  pdl_wait();

  // ------------------------------------------------------------ consumers
  const int nch = d / EC;
  const int j0 = (int)((long long)c * r / G), j1 = (int)((long long)(c + 1) * r / G);
  const int rpi = p1_rows_per_item(d);
  const int n_p1 = (j1 - j0 + rpi - 1) / rpi;
  const NeuronLayout<WT, ACT> NL(d);

  // FFN input u (fp16) for the owned column chunks, packed; chunks past the
  // row end hold zeros and read a clamped, valid address (branch-free loops)
  constexpr int UW = EC / 8;  // uint4 words of u per chunk
  uint4 uh[CPT][UW];
  int coff[CPT];  // clamped chunk index
#pragma unroll
  for (int q = 0; q < CPT; ++q) coff[q] = min(tid + q * kConsumers, nch - 1);
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
      const bool valid = tid + q * kConsumers < nch;
#pragma unroll
      for (int j = 0; j < UW; ++j) {
        uint32_t wd[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int e = coff[q] * EC + 8 * j + 2 * k;
          const __half lo = __float2half_rn(__fdiv_rn(x[e], den)), hi = __float2half_rn(__fdiv_rn(x[e + 1], den));
          wd[k] = valid ? ((uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16)) : 0u;
        }
        uh[q][j] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
      }
    }
  } else {
    const __half *uin = reinterpret_cast<const __half *>(a.in);
#pragma unroll
    for (int q = 0; q < CPT; ++q) {
      const bool valid = tid + q * kConsumers < nch;
#pragma unroll
      for (int j = 0; j < UW; ++j) {
        const uint4 v = ld_keep16(uin + coff[q] * EC + 8 * j);
        uh[q][j] = valid ? v : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
  // int4 dots take u in the (k, k+4) pair order of q8_pairs_biased, and the
  // chunk sums of u for the 1032 (= 1024 + 8) bias of the unpacked codes
  uint4 up4[CPT][UW];
  float usum[CPT];
#pragma unroll
  for (int q = 0; q < CPT; ++q) {
    usum[q] = 0.f;
#pragma unroll
    for (int j = 0; j < UW; ++j) {
      up4[q][j] = WT == W_INT4 ? pair_k4(uh[q][j]) : uh[q][j];
      if (WT == W_INT4) {
        const __half2 *hp = reinterpret_cast<const __half2 *>(&uh[q][j]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __half22float2(hp[k]);
          usum[q] += f.x;
          usum[q] += f.y;
        }
      }
    }
  }
  float y[CPT][EC];
#pragma unroll
  for (int q = 0; q < CPT; ++q)
#pragma unroll
    for (int e = 0; e < EC; ++e) y[q][e] = 0.f;

  // biases of this CTA's own neurons c + m G, one round trip
  for (int m = tid; m < nn; m += kConsumers) {
    const int i = c + m * G;
    S.own_pbias[m / kTN][m % kTN] = __ldg(a.p_bias + i);
    if (ACT == ACT_RELU) S.own_bup[m / kTN][m % kTN] = __ldg(a.b_up + i);
  }
  // clear the fired-bit words (CTA c clears words c, c + G, ...); the first
  // grid barrier orders this before any CTA sets bits
  if (a.idx != nullptr || a.count != nullptr)
    for (int w = c + tid * G; w < nwords; w += kConsumers * G) a.mask32[w] = 0u;

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

  // ---- P1 items: this CTA's slice of h (rows past the item alias row 0)
  for (int it = 0; it < n_p1 && alive; ++it) {
    int s;
    if (!(alive = wait_full(s))) break;
    const int rows = S.meta[s].n, jf = S.meta[s].first;
    float px[kMaxP1Rows], py[kMaxP1Rows];
#pragma unroll
    for (int q = 0; q < kMaxP1Rows; ++q) {
      px[q] = py[q] = 0.f;
      const __half *row = reinterpret_cast<const __half *>(S.ring[s]) + (size_t)(q < rows ? q : 0) * d;
#pragma unroll
      for (int cq = 0; cq < CPT; ++cq)
#pragma unroll
        for (int j = 0; j < UW; ++j)
          dot8_mixed(*reinterpret_cast<const uint4 *>(row + coff[cq] * EC + 8 * j), uh[cq][j], px[q], py[q]);
    }
    float part[kMaxP1Rows];
#pragma unroll
    for (int q = 0; q < kMaxP1Rows; ++q) part[q] = px[q] + py[q];
    warp_sum_n<kMaxP1Rows>(part);
    const int par = nr & 1;
    if (lane == 0) {
#pragma unroll
      for (int q = 0; q < kMaxP1Rows; ++q) S.red[par][warp][q] = part[q];
    }
    release(s);
    consumer_sync();
    ++nr;
    if (tid < rows) {
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
  const int pch = r / 8;
  for (int e = tid; e < r / 4; e += kConsumers)
    reinterpret_cast<float4 *>(S.h_s)[e] = __ldcg(reinterpret_cast<const float4 *>(a.h) + e);
  consumer_sync();
  // predictor columns of this lane: chunks lane + 32 kk (8 fp16 each)
  float hreg[4][8];
  int hoff[4];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int ch = lane + 32 * kk;
    hoff[kk] = min(ch, pch - 1);
#pragma unroll
    for (int e = 0; e < 8; ++e) hreg[kk][e] = (ch < pch) ? S.h_s[ch * 8 + e] : 0.f;
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
      // rows warp + 8 q of the tile: all of this warp's loads first, then the
      // dots, then one butterfly over the row sums
      const int kl = S.meta[s].first, rows = S.meta[s].n;
      constexpr int RPW = kTN / kConsumerWarps;
      unsigned b = 0u;
      uint4 wv[RPW][4];
#pragma unroll
      for (int q = 0; q < RPW; ++q) {
        const int row_i = warp + q * kConsumerWarps;
        const __half *row = reinterpret_cast<const __half *>(S.ring[s]) + (size_t)min(row_i, rows - 1) * r;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) wv[q][kk] = *reinterpret_cast<const uint4 *>(row + hoff[kk] * 8);
      }
      float sv[RPW];
#pragma unroll
      for (int q = 0; q < RPW; ++q) {
        float acc[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) acc[kk] = dot8_h2(wv[q][kk], hreg[kk]);
        sv[q] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
      }
      warp_sum_n<RPW>(sv);
#pragma unroll
      for (int q = 0; q < RPW; ++q) {
        const int row_i = warp + q * kConsumerWarps;
        if (row_i < rows && sv[q] + S.own_pbias[kl][row_i] > 0.f) b |= 1u << row_i;
      }
      if (lane == 0 && b) {
        atomicOr(&S.tbits[s], b);
        atomicOr(&S.own_bits[kl], b);
      }
      release(s);
      continue;
    }
    // IT_GATHER: neurons past the item alias neuron 0 and get a zero value
    const int ng = S.meta[s].n;
    const uint8_t *nd[kMaxGN];
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) nd[g] = S.ring[s] + (g < ng ? g : 0) * NL.bytes;
    float pu[kMaxGN], pg[kMaxGN];
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) {
      float ux = 0.f, uy = 0.f, gx = 0.f, gy = 0.f;
#pragma unroll
      for (int cq = 0; cq < CPT; ++cq) {
        if (WT == W_F16) {
          dot8_mixed(*reinterpret_cast<const uint4 *>(nd[g] + NL.up + coff[cq] * 16), uh[cq][0], ux, uy);
          if (ACT == ACT_SWIGLU)
            dot8_mixed(*reinterpret_cast<const uint4 *>(nd[g] + NL.gate + coff[cq] * 16), uh[cq][0], gx, gy);
        } else {
          // sum_k (q_k - 8) u_k = sum_k (1024 + q_k) u_k - 1032 sum_k u_k; the
          // products of two fp16 values are exact in fp32
          const float su = __half2float(*reinterpret_cast<const __half *>(nd[g] + NL.sup + (coff[cq] >> 1) * 2));
          const uint2 wu = *reinterpret_cast<const uint2 *>(nd[g] + NL.up + coff[cq] * 8);
          float x = 0.f, yv = 0.f;
          dot8_mixed(q8_pairs_biased(wu.x), up4[cq][0], x, yv);
          dot8_mixed(q8_pairs_biased(wu.y), up4[cq][1], x, yv);
          ux = fmaf(su, fmaf(-1032.f, usum[cq], x + yv), ux);
          if (ACT == ACT_SWIGLU) {
            const float sg = __half2float(*reinterpret_cast<const __half *>(nd[g] + NL.sgate + (coff[cq] >> 1) * 2));
            const uint2 wg = *reinterpret_cast<const uint2 *>(nd[g] + NL.gate + coff[cq] * 8);
            float x2 = 0.f, y2 = 0.f;
            dot8_mixed(q8_pairs_biased(wg.x), up4[cq][0], x2, y2);
            dot8_mixed(q8_pairs_biased(wg.y), up4[cq][1], x2, y2);
            gx = fmaf(sg, fmaf(-1032.f, usum[cq], x2 + y2), gx);
          }
        }
      }
      pu[g] = ux + uy;
      pg[g] = gx + gy;
    }
    const int par = nr & 1;
    {
      constexpr int NV = (ACT == ACT_SWIGLU) ? 2 * kMaxGN : kMaxGN;
      float pv[NV];
#pragma unroll
      for (int g = 0; g < kMaxGN; ++g) {
        pv[(ACT == ACT_SWIGLU) ? 2 * g : g] = pu[g];
        if (ACT == ACT_SWIGLU) pv[2 * g + 1] = pg[g];
      }
      warp_sum_n<NV>(pv);
      if (lane == 0) {
#pragma unroll
        for (int g = 0; g < kMaxGN; ++g) {
          S.red[par][warp][2 * g] = pv[(ACT == ACT_SWIGLU) ? 2 * g : g];
          S.red[par][warp][2 * g + 1] = (ACT == ACT_SWIGLU) ? pv[2 * g + 1] : 0.f;
        }
      }
    }
    // after this barrier every warp has also finished every earlier item,
    // so the fired bits of the neurons' tiles are complete
    consumer_sync();
    ++nr;
    // sum the 8 warps' partials: lane (g, w) = (lane / 8, lane % 8) loads
    // warp w's partial of neuron g, a 3-step butterfly over the 8 lanes of a
    // group adds them in a fixed order, and shuffles broadcast the sums
    float a_l = 0.f;  // on lanes 8g: value of neuron g
    {
      static_assert(kMaxGN * kConsumerWarps == 32, "one lane per (neuron, warp)");
      float vu = S.red[par][lane & 7][2 * (lane >> 3)];
      float vg = (ACT == ACT_SWIGLU) ? S.red[par][lane & 7][2 * (lane >> 3) + 1] : 0.f;
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) {
        vu += __shfl_xor_sync(0xffffffffu, vu, o);
        if (ACT == ACT_SWIGLU) vg += __shfl_xor_sync(0xffffffffu, vg, o);
      }
      // lanes 8g hold neuron g's sums: membership and activation there
      const int g_l = lane >> 3;
      if ((lane & 7) == 0 && g_l < ng) {
        const int m = S.meta[s].ids[g_l];  // own index: neuron c + m G
        const int kl = m / kTN;
        if ((S.own_bits[kl] >> (m % kTN)) & 1u) {
          if (ACT == ACT_RELU)
            a_l = fmaxf(vu + S.own_bup[kl][m % kTN], 0.f);
          else
            a_l = silu(vg) * vu;
        }
      }
    }
    // down-projection rows: y += a_g * W2T_g (every thread, its own chunks).
    // The rows of all the item's neurons are loaded first (neurons past the
    // item alias neuron 0); a_g is the same in every thread, so skipping the
    // zeros never diverges.
    float agv[kMaxGN];
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) agv[g] = __shfl_sync(0xffffffffu, a_l, 8 * g);
    constexpr int DW = WT == W_F16 ? 4 : 2;  // 32-bit words of a down chunk
    uint32_t wdn[kMaxGN][CPT][DW];
    float sdn[kMaxGN][CPT];
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g)
#pragma unroll
      for (int cq = 0; cq < CPT; ++cq) {
        if (WT == W_F16) {
          const uint4 v = *reinterpret_cast<const uint4 *>(nd[g] + NL.down + coff[cq] * 16);
          wdn[g][cq][0] = v.x;
          wdn[g][cq][1] = v.y;
          wdn[g][cq][DW - 2] = v.z;
          wdn[g][cq][DW - 1] = v.w;
          sdn[g][cq] = 1.f;
        } else {
          const uint2 v = *reinterpret_cast<const uint2 *>(nd[g] + NL.down + coff[cq] * 8);
          wdn[g][cq][0] = v.x;
          wdn[g][cq][DW - 1] = v.y;
          sdn[g][cq] = __half2float(*reinterpret_cast<const __half *>(nd[g] + NL.sdown + (coff[cq] >> 1) * 2));
        }
      }
#pragma unroll
    for (int g = 0; g < kMaxGN; ++g) {
      const float ag = agv[g];
      if (g >= ng || ag == 0.f) continue;
#pragma unroll
      for (int cq = 0; cq < CPT; ++cq) {
        if (WT == W_F16) {
          float w[8];
          h8_to_f8(make_uint4(wdn[g][cq][0], wdn[g][cq][1], wdn[g][cq][DW - 2], wdn[g][cq][DW - 1]), w);
#pragma unroll
          for (int e = 0; e < 8; ++e) y[cq][e] = fmaf(ag, w[e], y[cq][e]);
        } else {
          const float sd = sdn[g][cq];
          const uint2 wq = make_uint2(wdn[g][cq][0], wdn[g][cq][DW - 1]);
          const float as = ag * sd;
          // (q - 8) exactly, as the pairs (j, j + 4) of each 8-element word
          const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
          const uint4 p0 = q8_pairs_biased(wq.x), p1 = q8_pairs_biased(wq.y);
          const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int kq = 0; kq < 8; ++kq) {
            const __half2 hv = __hsub2(*reinterpret_cast<const __half2 *>(&pw[kq]), off);
            const float2 v = __half22float2(hv);
            const int e = (kq >> 2) * 8 + (kq & 3);  // elements e and e + 4 of the chunk
            y[cq][e] = fmaf(as, v.x, y[cq][e]);
            y[cq][e + 4] = fmaf(as, v.y, y[cq][e + 4]);
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
    if (col < c1) {
      constexpr int kMaxPer = 40;  // G <= 320
      float v[kMaxPer];
#pragma unroll
      for (int q = 0; q < kMaxPer; ++q) {
        const int cc = grp + q * kConsumerWarps;
        v[q] = (cc < G) ? ld_cg(a.partial + (size_t)cc * d + col) : 0.f;
      }
#pragma unroll
      for (int q = 0; q < kMaxPer; ++q) sum += v[q];
    }
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

  // ---- ascending active ids (optional): CTA c writes the ids of words
  // [c * tpc, (c + 1) * tpc) after the popcount of all earlier words
  if (a.idx != nullptr || a.count != nullptr) {
    const int tpc = (nwords + G - 1) / G;
    const int t0 = min(nwords, c * tpc), t1 = min(nwords, t0 + tpc);
    int before = 0, total = 0;
    for (int t = tid; t < nwords; t += kConsumers) {
      const int pc = __popc(__ldcg(a.mask32 + t));
      total += pc;
      if (t < t0) before += pc;
    }
    before = __reduce_add_sync(0xffffffffu, before);
    total = __reduce_add_sync(0xffffffffu, total);
    if (lane == 0) {
      S.iscan[warp] = before;
      S.dred[warp] = (double)total;
    }
    consumer_sync();
    if (tid == 0) {
      int b = 0, tt = 0;
      for (int w = 0; w < kConsumerWarps; ++w) {
        b += S.iscan[w];
        tt += (int)S.dred[w];
      }
      if (c == 0 && a.count) a.count[0] = tt;
      if (a.idx) {
        int pos = b;
        for (int t = t0; t < t1; ++t) {
          unsigned bits = __ldcg(a.mask32 + t);
          while (bits) {
            const int bit = __ffs(bits) - 1;
            bits &= bits - 1u;
            a.idx[pos++] = t * kTN + bit;
          }
        }
      }
    }
  }
}

}  // namespace fused
}  // namespace pi
