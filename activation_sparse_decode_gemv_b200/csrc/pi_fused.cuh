// pi_fused.cuh -- one persistent kernel per layer for the batch-1 decode step
// (PowerInfer summary page: Summary, per-layer predictor and neuron-level
// sparse kernels; Interesting ideas I1 hot/cold reordering, I4 kernels that
// read the rows of the active neurons directly).
//
// Grid: one CTA per SM, launched cooperatively (all CTAs co-resident).
// Block: 16 consumer warps + 1 producer warp.  The producer streams work items
// into a ring of 3 shared-memory slots with cp.async.bulk (TMA bulk copies)
// and mbarrier transaction counts; consumers process the slots in order:
//   P1 item     up to 8 rows of P1 owned by this CTA -> its slice of h = P1 u,
//               published to every CTA as tagged words (below)
//   P2 tile     32 predictor rows -> s = P2 h + bias, fire iff s > 0.  The
//               dot products run on the tensor cores (mma.sync m16n8k16):
//               A = the tile's rows, B = h split into h_hi = fp16(h) and
//               h_lo = fp16(h - h_hi) as the first two of the 8 columns, so
//               s = D[:,0] + D[:,1] carries h to about 22 bits.  Each warp
//               takes one sixteenth of the rank and leaves its partial sums
//               in shared memory; the producer, which waits for the slot
//               anyway, adds them in warp order and sets the fired bits, so a
//               tile costs the consumers neither a barrier nor an atomic.
//   GATHER      up (+gate) and down rows of 1-4 neurons: dot with u,
//               activation, then y += a * W2T_i in per-thread registers
//   DONE        end of the stream
// The producer "harvests" a tile when its slot's empty barrier completes
// (every consumer warp is done with it), appends the fired ids to its list
// and issues their gather rows; it keeps issuing P2 tiles meanwhile.  No L2
// prefetch runs ahead of the ring: prefetched predictor rows queued ahead of
// the latency-critical P1 and tile loads and made the step slower.
// Neurons are dealt round robin to the CTAs (neuron i to CTA i mod G),
// so every CTA gets the same mix of hot and cold neurons; CTA c's k-th tile
// holds its own neurons c + (32k + q) G, q < 32.  In dense hot-prefix mode the
// rows of a tile's prefix neurons are issued right after the tile, without
// waiting for its bits.
//
// Cross-CTA exchanges carry their own readiness: every value goes out as one
// 64-bit word (value bits, tag), stored and loaded with single-copy-atomic
// relaxed gpu-scope accesses.  The tag is the launch's epoch + 1; the epoch
// lives in the workspace, every CTA reads it after griddepcontrol.wait, and
// the rank-0 reducer advances it once its reduction has seen every CTA's
// partial (so every CTA has read it).  A reader polls until the tag matches,
// so publishing h or a partial of y costs one L2 round trip and no grid
// barrier.  After the stream every CTA publishes its fp32 partial of y; the
// CTAs that end their stream first (arrival ticket) each sum a column slice
// over all partials in CTA order (deterministic, no atomics on y) and write
// y (or add it to the residual x).
// Every wait is bounded (about 2 s); on expiry the kernel records
// PI_ERR_TIMEOUT in the workspace status word and completes.
#pragma once

#include <cuda.h>

#include <cstddef>

#include "pi_device.cuh"

namespace pi {
namespace fused {

constexpr int kConsumerWarps = 16;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kSlots = 3;
constexpr int kTN = 32;                      // neurons per predictor tile
constexpr int kMaxR = 1024;                  // predictor rank
// a slot holds one item: a predictor tile (32 rows of the rank, K-interleaved,
// plus the CTA's leftover row), up to 8 rows of P1, or the rows of 1-4 neurons
constexpr int kSlotBytes = (kTN + 1) * 2 * kMaxR;
constexpr int kMaxGN = 4;                    // neurons per gather item
constexpr int kMaxOwnTiles = 32;             // neurons per CTA <= 32 * 32
constexpr int kActCap = kMaxOwnTiles * kTN;  // capacity of the active-id list
constexpr int kMaxP1Rows = 8;                // P1 rows per item
constexpr int kMaxKs = kMaxR / 16 / kConsumerWarps;  // k16 steps of the rank per consumer warp
constexpr int kRedCols = 64;                 // columns of y each reducing CTA sums
constexpr int kRedBatch = 10;                // partials polled per batch by one reducing thread
constexpr unsigned long long kWaitNs = 2000000000ull;

enum ItemType : int { IT_P1 = 0, IT_P2 = 1, IT_GATHER = 2, IT_DONE = 3 };

struct SlotMeta {
  int type, n, first;
  int tslot;  // gather item of dense hot-prefix rows: buffer of their tile's partial scores; else -1
  int ids[kMaxGN];
};

struct Smem {
  uint8_t ring[kSlots][kSlotBytes];
  SlotMeta meta[kSlots];
  unsigned long long full[kSlots];
  unsigned long long empty[kSlots];
  int act[kActCap];                    // fired ids (index mode), producer-owned
  int tile_item[kMaxOwnTiles];         // item number each own tile was issued as
  float own_pbias[kMaxOwnTiles][kTN];  // predictor bias of this CTA's neurons
  float own_bup[kMaxOwnTiles][kTN];    // ReLU bias b1 of this CTA's neurons
  float h_s[kMaxR];                    // h, gathered from all CTAs
  // per-warp partial scores of own tile k, in buffer k % kSlots (tile k + 3
  // comes at least 3 items after tile k's last dense item, so it is not
  // issued before every warp is done with that item)
  float spart[kSlots][kConsumerWarps][kTN];
  float red[2][kConsumerWarps][2 * kMaxGN];
  double dred[kConsumerWarps];
  float fin[kConsumers / (kRedCols / 2)][kRedCols + 1];
  int iscan[kConsumerWarps];
  int slice;  // this CTA's reduction slice (its arrival rank at the stream end)
  volatile int abort_flag;
};

static_assert(offsetof(Smem, ring) == 0, "ring slots must start the shared block");
static_assert(kSlotBytes % 16 == 0, "bulk copies need 16-byte aligned slots");
static_assert(kSlotBytes % 128 == 0, "tensor copies need 128-byte aligned slots");
static_assert(sizeof(Smem) <= 227 * 1024, "shared memory per block");
static_assert(kConsumers * 2 * kRedBatch * 4 <= kSlots * kSlotBytes, "reduction stage fits the ring");

struct Args {
  // P2 as the 4D tensor (k % 8, m, k / 8, c) of neuron c + m G's element k,
  // m < f / G: one box {8, 32, r / 8, 1} is the 32 rows of a CTA's tile,
  // stored K-interleaved ([k / 8][row][k % 8], 16 bytes per row and chunk),
  // which ldmatrix reads without bank conflicts; rows past f / G read as 0
  CUtensorMap tm_p2;
  int p2_main;     // f / G (0: no main rows, and tm_p2 is not used)
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
  unsigned long long *hx;  // workspace [r] tagged h
  unsigned long long *px;  // workspace [G x d] tagged partials of y
  unsigned *epoch;         // workspace launch counter of the tags
  unsigned *ticket;        // workspace arrival counter of the reduction slices
  unsigned *mask32;  // workspace [ceil(f/32)] fired bits of neurons 32w..32w+31, when idx or count != nullptr
  unsigned *bar;     // workspace grid-barrier word (id lists only)
  int *status;
  int32_t *idx;    // optional ascending active ids [f]
  int32_t *count;  // optional [1]
  unsigned long long wait_ns;  // limit of every bounded wait
  int withhold;    // entry of h that is never published (-1: none); exercises the bounded waits
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
PI_DEV bool mbar_test(unsigned long long *b, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// bounded wait; false on timeout (status recorded).  It polls with
// test_wait and a short back-off: a thread parked by try_wait's suspend hint
// was measured to resume up to ~2 us after the phase completed, which delayed
// the producer's next copy by as much.  The fast path (phase already
// complete) is inline, the polling loop is out of line to keep the consumer
// loop small in the instruction cache.
__device__ __noinline__ bool mbar_wait_slow(unsigned long long *b, unsigned parity, int *status,
                                            unsigned long long limit) {
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (mbar_test(b, parity)) return true;
    if (globaltimer() - t0 > limit) {
      set_status(status, kStatusTimeout);
      return false;
    }
    __nanosleep(20);
  }
}
PI_DEV bool mbar_wait(unsigned long long *b, unsigned parity, int *status, unsigned long long limit) {
  if (mbar_test(b, parity)) return true;
  return mbar_wait_slow(b, parity, status, limit);
}
PI_DEV void bulk_g2s(void *dst, const void *src, unsigned bytes, unsigned long long *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
// 4D TMA box load at element coordinates (x0, x1, x2, x3) of a tensor map
// (a kernel parameter); elements outside the tensor read as zero
PI_DEV void tma_load_4d(void *dst, const CUtensorMap *tm, int x0, int x1, int x2, int x3, unsigned long long *bar) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], "
      "[%6];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<unsigned long long>(tm)), "r"(x0), "r"(x1), "r"(x2), "r"(x3), "r"(smem_u32(bar))
      : "memory");
}
PI_DEV void consumer_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
PI_DEV unsigned ld_acquire(const unsigned *p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
PI_DEV unsigned ld_relaxed_u32(const unsigned *p) {
  unsigned v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
PI_DEV void st_relaxed_u32(unsigned *p, unsigned v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---------------------------------------------------------------- tagged words
// (value, tag) as one 64-bit word: low half the value's bits, high half the tag
PI_DEV unsigned long long tagged(float v, unsigned tag) {
  return ((unsigned long long)tag << 32) | (unsigned long long)__float_as_uint(v);
}
PI_DEV float tagged_value(unsigned long long w) { return __uint_as_float((unsigned)(w & 0xffffffffull)); }
PI_DEV bool tag_is(unsigned long long w, unsigned tag) { return (unsigned)(w >> 32) == tag; }
PI_DEV void st_tagged(unsigned long long *p, unsigned long long w) {
  asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(w) : "memory");
}
PI_DEV void st_tagged2(unsigned long long *p, unsigned long long w0, unsigned long long w1) {
  asm volatile("st.relaxed.gpu.global.v2.b64 [%0], {%1, %2};" ::"l"(p), "l"(w0), "l"(w1) : "memory");
}
// two consecutive tagged words (16-byte aligned); each is its own
// single-copy-atomic 64-bit access
PI_DEV void ld_tagged2(const unsigned long long *p, unsigned long long &w0, unsigned long long &w1) {
  asm volatile("ld.relaxed.gpu.global.v2.b64 {%0, %1}, [%2];" : "=l"(w0), "=l"(w1) : "l"(p) : "memory");
}

// Grid-wide barrier, one thread per CTA (used only when the call asks for
// the global id list).  Every CTA adds 1 except CTA 0, which adds
// 2^31 - (G - 1): the word's top bit flips exactly when all G have arrived,
// and the low bits return to their previous value, so the word never needs
// resetting between barriers or launches.
PI_DEV bool grid_barrier(unsigned *bar, int G, int c, int *status, unsigned long long limit) {
  const unsigned inc = (c == 0) ? (0x80000000u - (unsigned)(G - 1)) : 1u;
  __threadfence();
  const unsigned old = atomicAdd(bar, inc);
  const unsigned long long t0 = globaltimer();
  for (;;) {
    if (((ld_acquire(bar) ^ old) & 0x80000000u) != 0u) return true;
    if (globaltimer() - t0 > limit) {
      set_status(status, kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

// ---------------------------------------------------------------- tensor-core helpers
PI_DEV void ldmatrix_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D += A B with A 16x16 fp16 (row-major fragments), B 16x8 fp16, D fp32
PI_DEV void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// fp16 pair (lo element first) of the high or low part of two fp32 values
PI_DEV uint32_t h_part_pair(float x0, float x1, int lo) {
  const __half a0 = __float2half_rn(x0), a1 = __float2half_rn(x1);
  __half v0 = a0, v1 = a1;
  if (lo) {
    v0 = __float2half_rn(x0 - __half2float(a0));
    v1 = __float2half_rn(x1 - __half2float(a1));
  }
  return (uint32_t)__half_as_ushort(v0) | ((uint32_t)__half_as_ushort(v1) << 16);
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

// k16 steps [ks0, ks1) of the rank taken by consumer warp w
PI_DEV void warp_ks(int r, int w, int &ks0, int &ks1) {
  const int ks = r / 16;
  ks0 = w * ks / kConsumerWarps;
  ks1 = (w + 1) * ks / kConsumerWarps;
}

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
  const unsigned p2b = (unsigned)r * 2u;
  const int M = a.p2_main;                       // rows of every CTA in the tensor map
  const int left_tile = (c < f - M * G) ? M / kTN : -1;  // tile holding this CTA's leftover row m = M
  constexpr int CPN = (ACT == ACT_SWIGLU ? 3 : 2) * (WT == W_INT4 ? 2 : 1);  // copies per neuron
  const bool want_mask = a.idx != nullptr || a.count != nullptr;
  const unsigned long long lim = a.wait_ns;
  unsigned pn = 0;   // items issued
  int k = 0;         // own tiles issued
  int hk = 0;        // own tiles harvested
  int act_tail = 0;  // fired own indices appended (index mode)
  int taken = 0;     // fired own indices issued as gather items
  bool ok = true;

  // own tile hk's partial scores are complete once its slot's empty phase
  // completed: lane q adds the 16 warps' partials of row q in warp order,
  // then the bias; fire iff s > 0
  auto harvest = [&]() {
    const int s = hk % kSlots;
    const int rows = min(kTN, nn - hk * kTN);
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) v += S.spart[s][w][lane];
    const unsigned bits = __ballot_sync(0xffffffffu, lane < rows && v + S.own_pbias[hk][lane] > 0.f);
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
    if (!mbar_wait(&S.empty[s], par, a.status, lim)) {
      if (lane == 0) S.abort_flag = 1;
      return false;
    }
    while (hk < k && (unsigned)S.tile_item[hk] + kSlots <= pn) harvest();
    return true;
  };
  // gather item: own indices ms[0..n); lane j issues copy j.  tslot: buffer
  // of the partial scores of the tile of dense hot-prefix rows (their bits
  // are not known yet), else -1
  auto issue_gather = [&](const int *ms, int n, int tslot) -> bool {
    int s;
    if (!acquire(s)) return false;
    if (lane == 0) {
      SlotMeta &m = S.meta[s];
      m.type = IT_GATHER;
      m.n = n;
      m.first = 0;
      m.tslot = tslot;
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
  // 2. predictor tiles, then gather rows.  Tiles go first: they decide which
  // rows are needed, so the last tile's fired neurons are not left for the
  // end of the stream
  while (ok) {
    while (hk < k && tile_done(hk)) harvest();
    if (k < nown) {
      const int rows = min(kTN, nn - k * kTN);
      int s;
      if (!(ok = acquire(s))) break;
      if (lane == 0) {
        S.meta[s].type = IT_P2;
        S.meta[s].n = rows;
        S.meta[s].first = k;
        S.tile_item[k] = (int)pn;
        const bool main = k * kTN < M, left = k == left_tile;
        mbar_arrive_tx(&S.full[s], (main ? (unsigned)kTN * p2b : 0u) + (left ? p2b : 0u));
        // one tensor copy for the tile's rows c + m G, m in [32k, min(32k + 32, M))
        if (main) tma_load_4d(S.ring[s], &a.tm_p2, 0, k * kTN, 0, c, &S.full[s]);
        // the leftover row c + M G (when c < f - M G), plain, after the box
        if (left) bulk_g2s(S.ring[s] + (size_t)kTN * p2b, a.p2 + (size_t)(c + M * G) * r, p2b, &S.full[s]);
      }
      __syncwarp();
      ++pn;
      // dense hot prefix: the tile's prefix neurons (the smallest ids), now
      const int ts = k % kSlots;
      int ms[kMaxGN], ng = 0;
      for (int q = 0; ok && q < rows; ++q) {
        if (c + (k * kTN + q) * G >= a.H) break;
        ms[ng++] = k * kTN + q;
        if (ng == GN) {
          ok = issue_gather(ms, ng, ts);
          ng = 0;
        }
      }
      if (ok && ng) ok = issue_gather(ms, ng, ts);
      ++k;
      continue;
    }
    if (taken < act_tail) {
      const int n = min(GN, act_tail - taken);
      ok = issue_gather(&S.act[taken], n, -1);
      taken += n;
      continue;
    }
    if (hk == nown) break;  // every tile harvested and every fired id issued
    // wait for the consumers to finish the oldest unharvested tile
    const unsigned it = (unsigned)S.tile_item[hk];
    if (!mbar_wait(&S.empty[it % kSlots], (it / kSlots) & 1u, a.status, lim)) {
      if (lane == 0) S.abort_flag = 1;
      ok = false;
      break;
    }
    harvest();
  }
  // 3. end of stream (also after an abort, so consumers stop)
  __threadfence();  // mask words visible before the consumers publish partials
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
__global__ void __launch_bounds__(kThreads, 1) decode_fused_kernel(const __grid_constant__ Args a) {
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
  const unsigned long long lim = a.wait_ns;

  if (tid == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kConsumerWarps);
    }
    S.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  // Programmatic dependent launch: the next step's grid may be scheduled
  // now, and its CTAs take SMs as this grid's CTAs leave.  The producer
  // streams weights only (P1 rows, P2 tiles, weight rows), which no earlier
  // kernel writes, so it starts at once; the consumers load this CTA's
  // biases (weights too), then wait for the preceding grid before reading
  // the input or touching the workspace.
  pdl_launch_dependents();
  if (warp == kConsumerWarps) {
    producer<WT, ACT>(S, a, c, G, lane);
    return;
  }
  constexpr int kBiasPer = kActCap / kConsumers;
  float pbv[kBiasPer], bupv[kBiasPer];
#pragma unroll
  for (int q = 0; q < kBiasPer; ++q) {
    const int m = tid + q * kConsumers;
    pbv[q] = bupv[q] = 0.f;
    if (m < nn) {
      pbv[q] = __ldg(a.p_bias + c + (size_t)m * G);
      if (ACT == ACT_RELU) bupv[q] = __ldg(a.b_up + c + (size_t)m * G);
    }
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
  unsigned tag = 0;
  if (a.stack) {
    tag = ld_relaxed_u32(a.epoch) + 1u;
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
    tag = ld_relaxed_u32(a.epoch) + 1u;  // in flight together with the loads of u
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

#pragma unroll
  for (int q = 0; q < kBiasPer; ++q) {
    const int m = tid + q * kConsumers;
    if (m < nn) {
      S.own_pbias[m / kTN][m % kTN] = pbv[q];
      S.own_bup[m / kTN][m % kTN] = bupv[q];
    }
  }
  // clear the fired-bit words (CTA c clears words c, c + G, ...); a grid
  // barrier orders this before any CTA sets bits
  if (a.idx != nullptr || a.count != nullptr) {
    for (int w = c + tid * G; w < nwords; w += kConsumers * G) a.mask32[w] = 0u;
    consumer_sync();
    if (tid == 0 && !grid_barrier(a.bar, G, c, a.status, lim)) S.abort_flag = 1;
  }

  unsigned n = 0;   // items consumed
  unsigned nr = 0;  // reductions done (parity of the red buffer)
  bool alive = true;
  auto wait_full = [&](int &s) -> bool {
    s = (int)(n % kSlots);
    if (!mbar_wait(&S.full[s], (n / kSlots) & 1u, a.status, lim)) {
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

  // ---- P1 items: this CTA's slice of h (rows past the item alias row 0),
  // published as tagged words
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
    if (tid < rows && jf + tid != a.withhold) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) t += S.red[par][w][tid];
      st_tagged(a.hx + jf + tid, tagged(t, tag));
    }
  }
  // ---- h of every CTA: each warp gathers the slice of the rank its tensor-
  // core steps use (lane: 4 consecutive entries), polling the tags
  int ks0, ks1;
  warp_ks(r, warp, ks0, ks1);
  if (alive) {
    // lane: entries e .. e + 3 (the warp's range is a multiple of 16 long).
    // Two rounds of loads stay in flight: a new round goes out before the
    // older one is checked, so a word published just after a round passed
    // the L2 is seen half a round trip later.
    const int e = ks0 * 16 + lane * 4;
    bool done = e >= ks1 * 16;
    unsigned long long wa[4], wb[4];
    if (!done) {
      ld_tagged2(a.hx + e, wa[0], wa[1]);
      ld_tagged2(a.hx + e + 2, wa[2], wa[3]);
    }
    // issue a round into wn, then check the older round wo
    auto round = [&](unsigned long long (&wo)[4], unsigned long long (&wn)[4]) {
      if (done) return;
      ld_tagged2(a.hx + e, wn[0], wn[1]);
      ld_tagged2(a.hx + e + 2, wn[2], wn[3]);
      if (tag_is(wo[0], tag) && tag_is(wo[1], tag) && tag_is(wo[2], tag) && tag_is(wo[3], tag)) {
        S.h_s[e] = tagged_value(wo[0]);
        S.h_s[e + 1] = tagged_value(wo[1]);
        S.h_s[e + 2] = tagged_value(wo[2]);
        S.h_s[e + 3] = tagged_value(wo[3]);
        done = true;
      }
    };
    // lane 0's clock decides for the warp, so the warp leaves together
    const unsigned long long t0 = globaltimer();
    auto expired = [&]() -> bool { return __shfl_sync(0xffffffffu, globaltimer() - t0 > lim ? 1 : 0, 0) != 0; };
    for (;;) {
      round(wa, wb);
      if (__all_sync(0xffffffffu, done)) break;
      round(wb, wa);
      if (__all_sync(0xffffffffu, done)) break;
      if (expired()) {
        set_status(a.status, kStatusTimeout);
        S.abort_flag = 1;
        alive = false;
        break;
      }
    }
    __syncwarp();
  }
  // a warp that gave up makes the whole CTA skip the stream, so that every
  // consumer warp meets the same block barriers
  consumer_sync();
  alive = alive && !S.abort_flag;
  // B fragments of this warp's k16 steps: lanes 0-3 hold h_hi, lanes 4-7
  // h_lo (columns 0 and 1 of B); every other lane holds zeros
  uint32_t hb[kMaxKs][2];
#pragma unroll
  for (int i = 0; i < kMaxKs; ++i) {
    hb[i][0] = hb[i][1] = 0u;
    if (lane < 8 && ks0 + i < ks1 && alive) {
      const int k0 = (ks0 + i) * 16 + 2 * (lane & 3), lo = lane >> 2;
      hb[i][0] = h_part_pair(S.h_s[k0], S.h_s[k0 + 1], lo);
      hb[i][1] = h_part_pair(S.h_s[k0 + 8], S.h_s[k0 + 9], lo);
    }
  }
  const int nks = ks1 - ks0;
  // ldmatrix row addresses in the K-interleaved tile ([k / 8][row][k % 8],
  // 16 bytes per row and chunk): lane L reads row L % 16 at k chunk
  // 2 ks + L / 16; one k16 step is 2 chunks of 32 rows (1 KB), a 16-row half
  // 256 bytes.  The CTA's leftover row (c < f - M G) sits, plain, after the
  // box of its tile; the two lanes that read its position read it there.
  const uint32_t a_off = ((uint32_t)(2 * ks0 + (lane >> 4)) * (uint32_t)kTN + (uint32_t)(lane & 15)) * 16u;
  const int M = a.p2_main;
  const int left_tile = (c < f - M * G) ? M / kTN : -1;
  const int left_pos = M % kTN;
  const bool left_lane = (lane & 15) == (left_pos & 15);
  const uint32_t left_off = (uint32_t)kTN * 2u * (uint32_t)r + (uint32_t)(2 * ks0 + (lane >> 4)) * 16u;

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
      // this warp's k16 steps of both 16-row halves of the tile
      const int kl = S.meta[s].first;
      float acc[2][4];
#pragma unroll
      for (int mb = 0; mb < 2; ++mb)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mb][e] = 0.f;
      const uint32_t slot = smem_u32(S.ring[s]);
      const bool lt = kl == left_tile && left_lane;
#pragma unroll
      for (int i = 0; i < kMaxKs; ++i) {
        if (i < nks) {
#pragma unroll
          for (int mb = 0; mb < 2; ++mb) {
            uint32_t af[4];
            const uint32_t ad = (lt && mb == (left_pos >> 4)) ? slot + left_off + (uint32_t)i * 32u
                                                              : slot + a_off + (uint32_t)mb * 256u + (uint32_t)i * 1024u;
            ldmatrix_x4(ad, af);
            mma_16816(acc[mb], af, hb[i][0], hb[i][1]);
          }
        }
      }
      // lanes 4g hold rows g and g + 8 of each half: s = D[.,0] + D[.,1]
      if ((lane & 3) == 0) {
        const int g = lane >> 2, b = kl % kSlots;
        S.spart[b][warp][g] = acc[0][0] + acc[0][1];
        S.spart[b][warp][g + 8] = acc[0][2] + acc[0][3];
        S.spart[b][warp][g + 16] = acc[1][0] + acc[1][1];
        S.spart[b][warp][g + 24] = acc[1][2] + acc[1][3];
      }
      release(s);
      continue;
    }
    // IT_GATHER: neurons past the item alias neuron 0 and get a zero value.
    // Index-mode items hold fired neurons only; for dense hot-prefix rows the
    // lanes 8g work out membership from their tile's partial scores (same
    // sum, same order as the producer's) after the barrier below, when every
    // warp has written its partials of that tile
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
    // sum the 16 warps' partials: lane (g, w) = (lane / 8, lane % 8) adds the
    // partials of neuron g from warps w and w + 8, a 3-step butterfly over the
    // 8 lanes of a group adds those in a fixed order, and shuffles broadcast
    // the sums
    float a_l = 0.f;  // on lanes 8g: value of neuron g
    {
      static_assert(kMaxGN * kConsumerWarps == 64, "one lane per neuron and warp pair");
      float vu = S.red[par][lane & 7][2 * (lane >> 3)] + S.red[par][(lane & 7) + 8][2 * (lane >> 3)];
      float vg = (ACT == ACT_SWIGLU)
                     ? S.red[par][lane & 7][2 * (lane >> 3) + 1] + S.red[par][(lane & 7) + 8][2 * (lane >> 3) + 1]
                     : 0.f;
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
        bool member = true;
        const int ts = S.meta[s].tslot;
        if (ts >= 0) {
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) v += S.spart[ts][w][m % kTN];
          member = v + S.own_pbias[kl][m % kTN] > 0.f;
        }
        if (member) {
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

  // arrival ticket, in flight while the partial goes out: the CTAs that end
  // their stream first sum the slices of y, so a heavily loaded CTA does not
  // also hold one back (whichever CTA sums a slice adds the partials in CTA
  // order, so y does not depend on the arrival order)
  constexpr int kTicketThread = kConsumers - 1;  // fewest column chunks
  unsigned ticket_raw = 0u;
  if (tid == kTicketThread) ticket_raw = atomicAdd(a.ticket, 1u);
  if (S.abort_flag && tid == 0) {
    // a wait gave up: let any bulk copy still in flight into this CTA's
    // shared memory land before the CTA can exit (bounded, about 1 ms)
    const unsigned long long t0 = globaltimer();
    while (globaltimer() - t0 < 1000000ull) __nanosleep(1000);
  }
  // ---- publish this CTA's partial of y as tagged words (after an abort too,
  // so that the other CTAs' reductions complete)
  if (a.idx != nullptr || a.count != nullptr) __threadfence();  // mask words before the partials
  {
    unsigned long long *pc = a.px + (size_t)c * d;
#pragma unroll
    for (int cq = 0; cq < CPT; ++cq) {
      const int ch = tid + cq * kConsumers;
      if (ch < nch) {
#pragma unroll
        for (int e = 0; e < EC; e += 2)
          st_tagged2(pc + (size_t)ch * EC + e, tagged(y[cq][e], tag), tagged(y[cq][e + 1], tag));
      }
    }
  }

  // ---- reduction.  The CTAs with the first R arrival ranks (R =
  // ceil(d / kRedCols)) each sum the slice of kRedCols columns of their rank
  // over all G partials; the others leave now, so the next launch's CTAs can
  // take their SMs and start streaming weights while the reduction runs (the
  // id lists, when asked for, need every CTA).  The rank is the ticket mod
  // G, a permutation of 0..G-1 within a launch whatever the counter held;
  // the holder of rank G - 1 takes G back off, so the counter stays below 2G.
  // Thread (grp, p) = (tid / 32, tid % 32) takes the column pair 2p of the
  // slice from CTAs grp, grp + 16, ... (in that order), then the 16 group
  // sums are added in group order: a fixed order, so y is deterministic.
  if (tid == kTicketThread) {
    const unsigned t = ticket_raw % (unsigned)G;
    if (t == (unsigned)G - 1u) atomicSub(a.ticket, (unsigned)G);
    S.slice = (int)t;
  }
  consumer_sync();
  const int sl = S.slice;
  const bool want_ids = a.idx != nullptr || a.count != nullptr;
  const int n_red = (d + kRedCols - 1) / kRedCols;
  if (sl >= n_red && !want_ids) return;
  if (sl < n_red) {
    constexpr int kGroups = kConsumers / (kRedCols / 2);
    const int pr = tid % (kRedCols / 2), grp = tid / (kRedCols / 2);
    const int col = sl * kRedCols + 2 * pr;
    float s0 = 0.f, s1 = 0.f;
    bool timed_out = false;
    if (col < d) {
      // batches of kRedBatch partials: all loads of a batch go out before any
      // tag is checked; the values wait in this thread's stage in the (now
      // idle) ring until the batch is complete, then add in CTA order
      float *stage = reinterpret_cast<float *>(S.ring[0]) + (size_t)tid * 2 * kRedBatch;
      for (int qb = 0; grp + qb * kGroups < G; qb += kRedBatch) {
        unsigned pending = 0u;
#pragma unroll
        for (int q = 0; q < kRedBatch; ++q)
          if (grp + (qb + q) * kGroups < G) pending |= 1u << q;
        const unsigned all = pending;
        const unsigned long long t0 = globaltimer();
        while (pending && !timed_out) {
          unsigned long long w0[kRedBatch], w1[kRedBatch];
#pragma unroll
          for (int q = 0; q < kRedBatch; ++q)
            if ((pending >> q) & 1u) ld_tagged2(a.px + (size_t)(grp + (qb + q) * kGroups) * d + col, w0[q], w1[q]);
#pragma unroll
          for (int q = 0; q < kRedBatch; ++q) {
            if (((pending >> q) & 1u) && tag_is(w0[q], tag) && tag_is(w1[q], tag)) {
              stage[2 * q] = tagged_value(w0[q]);
              stage[2 * q + 1] = tagged_value(w1[q]);
              pending &= ~(1u << q);
            }
          }
          if (pending) {
            if (globaltimer() - t0 > lim) {
              set_status(a.status, kStatusTimeout);
              timed_out = true;
            } else {
              __nanosleep(32);
            }
          }
        }
        for (int q = 0; q < kRedBatch; ++q) {
          if (((all >> q) & 1u) && !((pending >> q) & 1u)) {
            s0 += stage[2 * q];
            s1 += stage[2 * q + 1];
          }
        }
      }
    }
    S.fin[grp][2 * pr] = s0;
    S.fin[grp][2 * pr + 1] = s1;
    consumer_sync();
    if (tid < kRedCols && sl * kRedCols + tid < d) {
      float t = S.fin[0][tid];
#pragma unroll
      for (int g = 1; g < kGroups; ++g) t += S.fin[g][tid];
      const int oc = sl * kRedCols + tid;
      a.out[oc] = (a.stack || a.accumulate) ? a.out[oc] + t : t;
    }
  }
  // every CTA has read the epoch (its partial carries this launch's tag):
  // the rank-0 reducer advances it for the next launch on this workspace
  if (sl == 0 && tid == 0) st_relaxed_u32(a.epoch, tag);

  // ---- ascending active ids (optional): after a grid barrier, CTA c writes
  // the ids of words [c * tpc, (c + 1) * tpc) after the popcount of all
  // earlier words
  if (a.idx != nullptr || a.count != nullptr) {
    consumer_sync();
    if (tid == 0) {
      if (!grid_barrier(a.bar, G, c, a.status, lim)) S.abort_flag = 1;
    }
    consumer_sync();
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
