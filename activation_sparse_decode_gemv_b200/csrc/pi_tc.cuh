// pi_tc.cuh -- tensor-core (tcgen05) path for token batches of 16..32.
//
// At batch >= 16 the union of the tokens' predicted sets covers nearly every
// neuron, so each 128-neuron block is a dense contraction with the 16..32
// token columns as the MMA's N.  Four persistent kernels run the step, each
// on one CTA per SM with a stream-K split of its (tile, K-step) units so that
// all SMs end together:
//
//   pred_h  : h^T[r x N]  = P1 u^T               (A = P1, K = d)
//   pred_s  : s^T[f x N]  = P2 (h_hi + h_lo)^T   (A = P2, K = r) + bias,
//             thresholded into the per-token mask words
//   ffn_up  : a^T         = act(W_up/gate u^T) on every 128-neuron tile that
//             holds a predicted neuron of some token; zero where the token
//             did not predict the neuron        (A = weight rows, K = d)
//   ffn_down: y^T[d x N]  = W2T^T a^T over those tiles (A = W2T, MN-major)
//
// Row data moves by TMA (2D tensor maps, one 16 KB box of 128 rows per
// copy).  fp16 boxes land 128B-swizzled, which is the canonical UMMA layout,
// so the MMA reads them in place.  int4 boxes (packed nibbles + the group
// scales) are dequantised by eight worker warps into tensor memory (A operand
// of the MMA) for the up/gate GEMM, or into a canonical shared-memory tile
// for the down GEMM.  One thread issues the MMAs; the worker warps also run
// the epilogues.
//
// Token operands are "images": per 16-deep K block, 1 KB holding the 32 token
// rows in the canonical no-swizzle K-major layout (core matrices of 8 tokens
// x 8 K, 16-byte rows).  Padding tokens and K beyond the row are zero, and
// TMA fills rows or columns outside a matrix with zeros, so padded MMA work
// adds exact zeros.
//
// Stream-K: a kernel's W = tiles x steps units are split into contiguous
// spans over min(G, W) CTAs.  A tile whose steps span several CTAs is
// finished by the last CTA to arrive (per-tile counter): it adds the pieces'
// fp32 partials in K order, so the result does not depend on timing.
// Counters reset themselves.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "pi_device.cuh"

namespace pi {
namespace tc {

constexpr int kN = 32;        // MMA N: token columns (batches of 16..32 are zero-padded)
constexpr int kM = 128;       // MMA M: rows of a tile
constexpr int kBlk = 1024;    // bytes of one 16-deep K block of a token image
// warp 0 producer, warp 1 MMA issuer, warps 2.. workers (8, or 16 for int4 dequant)
constexpr int kThreads = 320;      // 8 worker warps
constexpr int kMaxThreads = 576;   // 16 worker warps
constexpr int kSmemBudget = 216 * 1024;
constexpr int kPartFloats = 128 * 64;  // largest per-piece partial (floats)
constexpr int kDownTileD = 256;        // d positions per down-projection tile (two M=128 MMAs)
constexpr int kDownStepK = 64;         // neurons per down-projection step
constexpr int kMaxTiles = 1024;        // 128-neuron tiles the ffn kernels can list (d_ffn <= 131072)
constexpr int kImgStep = 128;          // token images are padded to a multiple of 128 in K
constexpr uint32_t kSw128 = 2;         // UMMA descriptor layout code of the 128-byte swizzle
constexpr int kMaxSlots = 12;          // deepest ring (bytes in flight per SM are what hide the latency)
constexpr unsigned long long kWaitNs = 2000000000ull;

enum Kind { K_P1 = 0, K_P2 = 1, K_UP = 2 };

// ---------------------------------------------------------------- PTX helpers
PI_DEV uint32_t su32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
PI_DEV unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

PI_DEV void mbar_init(uint64_t *b, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(count) : "memory");
}
PI_DEV void mbar_arrive(uint64_t *b) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
PI_DEV void mbar_expect_tx(uint64_t *b, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes)
               : "memory");
}
// non-blocking test of the phase with the given parity
PI_DEV bool mbar_test(uint64_t *b, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// try_wait with a suspend-time hint: the thread is parked until the phase
// completes or the hint elapses, instead of spinning on the barrier
PI_DEV bool mbar_try(uint64_t *b, unsigned parity, unsigned hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity.  Gives up when another
// role of the CTA has aborted or after kWaitNs (recording a timeout).
__device__ __noinline__ bool mbar_wait_slow(uint64_t *b, unsigned parity, volatile int *abort_flag, int *status) {
  const unsigned long long t0 = now_ns();
  for (;;) {
    if (mbar_try(b, parity, 20000u)) return true;
    if (*abort_flag) return false;
    if (now_ns() - t0 > kWaitNs) {
      set_status(status, kStatusTimeout);
      *abort_flag = 1;
      return false;
    }
  }
}
PI_DEV bool mbar_wait(uint64_t *b, unsigned parity, volatile int *abort_flag, int *status) {
  if (mbar_test(b, parity)) return true;
  return mbar_wait_slow(b, parity, abort_flag, status);
}
// the same, agreed by the whole warp (lanes that see different outcomes all give up)
PI_DEV bool mbar_wait_warp(uint64_t *b, unsigned parity, volatile int *abort_flag, int *status) {
  return __all_sync(0xffffffffu, mbar_wait(b, parity, abort_flag, status));
}
// bounded barrier of the 256 worker threads on an mbarrier of count 256
PI_DEV bool workers_bar(uint64_t *b, unsigned &phase, volatile int *abort_flag, int *status) {
  mbar_arrive(b);
  const bool ok = mbar_wait_warp(b, phase, abort_flag, status);
  phase ^= 1u;
  return ok;
}

// 2D TMA tile load of the box at element coordinates (x, y) of a tensor map
// (a kernel parameter); rows or columns outside the tensor read as zero
PI_DEV void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(su32(bar))
      : "memory");
}

PI_DEV void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(su32(bar))
               : "memory");
}

PI_DEV void proxy_fence_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
PI_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
PI_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// tensor memory: allocation by one whole warp
PI_DEV void tmem_alloc(uint32_t *slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(slot)), "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
PI_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// UMMA shared-memory descriptor: start, leading and stride byte offsets,
// layout (0: no swizzle, kSw128: 128-byte swizzle with 1024-byte aligned atoms)
PI_DEV uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout = 0) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46) | ((uint64_t)layout << 61);
}
// instruction descriptor of kind::f16: fp16 A and B, fp32 accumulator, M x N
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

PI_DEV void mma_ts(uint32_t d, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
PI_DEV void mma_ss(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// arrive on b when every tcgen05 operation issued so far by this thread is done
PI_DEV void mma_commit(uint64_t *b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(b))
               : "memory");
}

PI_DEV void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
      "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
PI_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
PI_DEV void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

PI_DEV void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int j = 0; j < 8; ++j) v[j] = __uint_as_float(r[j]);
}
PI_DEV void tmem_st16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}

// byte offset of (token n, k) inside one 16-deep K block of a token image
PI_DEV uint32_t img_off(int n, int k) {
  return (uint32_t)((n >> 3) * 256 + (k >> 3) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// ---------------------------------------------------------------- int4 -> fp16 pairs
// One 32-bit word of packed nibbles (element 2j in the low nibble of byte j)
// to four fp16 pairs s * (q - 8), element 2c in the low half of column c.
// 0x6400 | q is the fp16 value 1024 + q; subtracting 1032 is exact and the
// product with the scale is the only rounding.
PI_DEV void q8_to_h4(uint32_t w, __half2 s2, uint32_t (&o)[4]) {
  const uint32_t lo = w & 0x0F0F0F0Fu;         // e0 e2 e4 e6 (bytes)
  const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // e1 e3 e5 e7
  const uint32_t t0 = __byte_perm(lo, hi, 0x5140);  // e0 e1 e2 e3
  const uint32_t t1 = __byte_perm(lo, hi, 0x7362);  // e4 e5 e6 e7
  const uint32_t k64 = 0x64646464u;
  const uint32_t p[4] = {__byte_perm(t0, k64, 0x4140), __byte_perm(t0, k64, 0x4342), __byte_perm(t1, k64, 0x4140),
                         __byte_perm(t1, k64, 0x4342)};
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    __half2 v = __hmul2(__hsub2(*reinterpret_cast<const __half2 *>(&p[c]), off), s2);
    o[c] = *reinterpret_cast<uint32_t *>(&v);
  }
}

// One 32-bit word of packed nibbles n0..n7 to the four fp16 pairs
// (n0, n4), (n1, n5), (n2, n6), (n3, n7), each s * (q - 8).  Pairing nibble j
// with nibble j + 4 needs only a shift and a masked OR per pair; the K order
// this gives (positions 2j, 2j+1 of an 8-block hold elements j, j+4) is
// matched by the permuted token image (u_image_kernel).
PI_DEV void q8_to_h4_paired(uint32_t w, __half2 s2, uint32_t (&o)[4]) {
  const __half2 off = __halves2half2(__ushort_as_half(0x6408), __ushort_as_half(0x6408));
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t p = ((w >> (4 * j)) & 0x000F000Fu) | 0x64006400u;
    __half2 v = __hmul2(__hsub2(*reinterpret_cast<const __half2 *>(&p), off), s2);
    o[j] = *reinterpret_cast<uint32_t *>(&v);
  }
}

// ---------------------------------------------------------------- stream-K
struct Span {
  long long u0, u1;  // this CTA's units [u0, u1)
};
PI_DEV Span span_of(long long W, int G, int c) { return Span{W * c / G, W * (c + 1) / G}; }
// CTA owning unit u
PI_DEV int owner_of(long long u, long long W, int G) { return (int)(((u + 1) * G + W - 1) / W) - 1; }

// ---------------------------------------------------------------- token image
// u [B x d] fp16 -> image of ceil(d/128)*8 blocks; tokens >= B and k >= d are
// 0.  img_perm (optional) receives the same image with every 8-element K
// block in the order 0 4 1 5 2 6 3 7 (the order of q8_to_h4_paired).
__global__ void __launch_bounds__(256) u_image_kernel(const __half *__restrict__ u, int B, int d,
                                                      unsigned char *__restrict__ img,
                                                      unsigned char *__restrict__ img_perm) {
  pdl_wait();
  pdl_launch_dependents();
  const int nblk = (d + kImgStep - 1) / kImgStep * 8;
  const int per_tok = nblk * 2;  // 16-byte pieces per token row of the image
  const int total = kN * per_tok;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < total; c += gridDim.x * blockDim.x) {
    const int n = c / per_tok, j = c - n * per_tok;
    const int blk = j >> 1, kh = j & 1;
    const int k0 = blk * 16 + kh * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < B && k0 < d) v = *reinterpret_cast<const uint4 *>(u + (size_t)n * d + k0);
    *reinterpret_cast<uint4 *>(img + (size_t)blk * kBlk + img_off(n, kh * 8)) = v;
    if (img_perm)
      *reinterpret_cast<uint4 *>(img_perm + (size_t)blk * kBlk + img_off(n, kh * 8)) =
          make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632), __byte_perm(v.y, v.w, 0x5410),
                     __byte_perm(v.y, v.w, 0x7632));
  }
}

// ---------------------------------------------------------------- shared pieces
struct TcCtrl {
  uint64_t full[kMaxSlots], empty[kMaxSlots];
  uint64_t afull[2], afree[2], accfull[2], accfree[2];
  uint64_t wbar;  // the 256 worker threads' barrier (stream-K fix-up)
  uint32_t tmem;
  int abort_flag;
  int is_last;
  int n_tiles;    // tiles listed in tlist
  int wcnt[kMaxThreads / 32];
  int tlist[kMaxTiles];  // ffn kernels: 128-neuron tiles holding a predicted neuron
};
constexpr int kCtrlBytes = 5120;
static_assert(sizeof(TcCtrl) <= kCtrlBytes, "control block");

// nw: worker warps.  empty_count: arrivals that free a ring slot (1: the
// MMA's commit; nw + 1: the worker warps that read the slot and the commit)
template <int NSLOT>
PI_DEV void ctrl_init(TcCtrl &C, unsigned nw, unsigned empty_count) {
  for (int s = 0; s < NSLOT; ++s) {
    mbar_init(&C.full[s], 1);  // the producer's expect_tx; TMA completes the bytes
    mbar_init(&C.empty[s], empty_count);
  }
  for (int b = 0; b < 2; ++b) {
    mbar_init(&C.afull[b], nw);
    mbar_init(&C.afree[b], 1);
    mbar_init(&C.accfull[b], 1);
    mbar_init(&C.accfree[b], nw);
  }
  mbar_init(&C.wbar, nw * 32);
  C.abort_flag = 0;
  C.is_last = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// All threads: list the 128-neuron tiles that hold a set bit of the union
// words (4 words per tile: the OR of the tokens' mask words), in ascending
// order, into C.tlist / C.n_tiles.
PI_DEV void list_tiles(TcCtrl &C, const uint32_t *uwords, int nwords, int n_all) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, nthreads = blockDim.x;
  int base = 0;
  for (int t0 = 0; t0 < n_all; t0 += nthreads) {
    const int t = t0 + tid;
    bool act = false;
    if (t < n_all) {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (4 * t + k < nwords) act |= __ldcg(uwords + 4 * t + k) != 0u;
    }
    const unsigned bal = __ballot_sync(0xffffffffu, act);
    if (lane == 0) C.wcnt[warp] = __popc(bal);
    __syncthreads();
    int off = base;
    for (int w = 0; w < warp; ++w) off += C.wcnt[w];
    if (act) C.tlist[off + __popc(bal & ((1u << lane) - 1u))] = t;
    int tot = 0;
    for (int w = 0; w < nthreads / 32; ++w) tot += C.wcnt[w];
    base += tot;
    __syncthreads();
  }
  if (tid == 0) C.n_tiles = base;
  __syncthreads();
}

// Stream-K fix-up for one worker thread's NV accumulator values of a piece
// that does not cover its whole tile (G: the CTAs the units were split
// over).  Publishes the piece; the CTA whose piece arrives last sums all
// pieces in K order into v and returns true.  *ok turns false when a bounded
// wait gave up.
template <int NV>
PI_DEV bool stream_k_finish(float (&v)[NV], float *part, int *ctr, int tile, long long SK, long long W, int G,
                            int cta, long long u0, int w, int lane, TcCtrl &C, unsigned &wphase,
                            volatile int *abort_flag, int *status, bool *ok) {
  const int slot = (int)(u0 / SK) == tile ? 0 : 1;
  float *mine = part + ((size_t)cta * 2 + slot) * kPartFloats;
#pragma unroll
  for (int j = 0; j < NV; ++j) mine[(w * NV + j) * 32 + lane] = v[j];
  __threadfence();
  if (!workers_bar(&C.wbar, wphase, abort_flag, status)) {
    *ok = false;
    return false;
  }
  const long long tu0 = (long long)tile * SK, tu1 = tu0 + SK - 1;
  const int c0 = owner_of(tu0, W, G), c1 = owner_of(tu1, W, G);
  if (w == 0 && lane == 0) {
    __threadfence();
    const int old = atomicAdd(ctr + tile, 1);
    const int lastp = old == c1 - c0;
    if (lastp) ctr[tile] = 0;
    __threadfence();
    C.is_last = lastp;
  }
  if (!workers_bar(&C.wbar, wphase, abort_flag, status)) {
    *ok = false;
    return false;
  }
  if (!C.is_last) return false;
  // pieces are loaded PB at a time (independent loads in flight) and added in K order
  constexpr int PB = NV >= 16 ? 2 : 4;
  float acc[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) acc[j] = 0.f;
  for (int c = c0; c <= c1; c += PB) {
    float t[PB][NV];
#pragma unroll
    for (int k = 0; k < PB; ++k) {
      const int cc = c + k;
      if (cc <= c1 && cc != cta) {
        const int cslot = (int)(span_of(W, G, cc).u0 / SK) == tile ? 0 : 1;
        const float *pp = part + ((size_t)cc * 2 + cslot) * kPartFloats;
#pragma unroll
        for (int j = 0; j < NV; ++j) t[k][j] = __ldcg(pp + (w * NV + j) * 32 + lane);
      } else {
#pragma unroll
        for (int j = 0; j < NV; ++j) t[k][j] = v[j];
      }
    }
#pragma unroll
    for (int k = 0; k < PB; ++k)
      if (c + k <= c1)
#pragma unroll
        for (int j = 0; j < NV; ++j) acc[j] += t[k][j];
  }
#pragma unroll
  for (int j = 0; j < NV; ++j) v[j] = acc[j];
  return true;
}

// Releases tensor memory.  Every MMA has finished by then: the workers wait
// for the commit that follows the last MMA of each piece, the last piece
// included (a CTA that gave up on a bounded wait skips that guarantee).
PI_DEV void teardown(int warp, uint32_t tmem, uint32_t ncols) {
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

// ---------------------------------------------------------------- row GEMMs: pred_h, pred_s, ffn_up
struct RowArgs {
  CUtensorMap tm0, tm1;         // row data of matrix 0 / 1: fp16 [rows x K] (box 64 x 128) or
                                // packed int4 bytes [rows x K/2] (box 128 x 128)
  CUtensorMap ts0, ts1;         // int4 scale bytes [rows x K/16] (box 16 x 128)
  int nrows;                    // rows of the matrices
  int K;                        // row length (elements)
  const unsigned char *img0;    // B operand image (u, or h_hi)
  const unsigned char *img1;    // pred_s: h_lo image
  const float *bias;            // pred_s: predictor bias; ffn_up ReLU: b_up
  const uint32_t *mask;         // ffn_up: per-token mask words [B x nwords]
  uint32_t *mask_out;           // pred_s: per-token mask words [B x nwords]
  uint32_t *uwords;             // pred_h: zeroed; pred_s: OR of the tokens' mask words; ffn_up: read
  int nwords, B;
  unsigned char *out0, *out1;   // pred_h: h_hi / h_lo images; ffn_up: a image
  float *part;                  // stream-K partials [G x 2 x kPartFloats]
  int *ctr;                     // per-tile arrival counters (zero between launches)
  int *status;
};

template <int KIND, int WT, int ACT>
struct RowShape {
  static constexpr int NMAT = (KIND == K_UP && ACT == ACT_SWIGLU) ? 2 : 1;
  static constexpr int NIMG = KIND == K_P2 ? 2 : 1;
  static constexpr bool Q4 = WT == W_INT4;
  static constexpr int STEPK = Q4 ? 256 : 64;       // K per unit
  static constexpr int ABOX = 16384;                // one box: 128 rows x 128 bytes
  static constexpr int SBOX = Q4 ? 2048 : 0;        // int4 scales: 128 rows x 16 bytes
  static constexpr int IMGB = NIMG * (STEPK / 16) * kBlk;
  static constexpr int SC_OFF = NMAT * ABOX;
  static constexpr int IMG_OFF = NMAT * (ABOX + SBOX);
  static constexpr int SLOTB = (IMG_OFF + IMGB + 1023) / 1024 * 1024;
  static constexpr int NSLOT_FIT = kSmemBudget / SLOTB;
  static constexpr int NSLOT = NSLOT_FIT > kMaxSlots ? kMaxSlots : NSLOT_FIT;
  static constexpr int TX = IMG_OFF + IMGB;         // bytes landing per unit
  static constexpr int CTRL_OFF = NSLOT * SLOTB;
  static constexpr int SMEM = CTRL_OFF + kCtrlBytes + 1024;  // + alignment slack
  static constexpr int ACC_COLS = NMAT * kN;        // per accumulator buffer
  static constexpr int A_COLS = NMAT * 64;          // int4: per tensor-memory A buffer (128 K)
  static constexpr uint32_t TMEM_COLS = Q4 ? 512 : 128;
  static constexpr int NW = 8;                      // worker warps
  static constexpr int THREADS = 64 + 32 * NW;
  static constexpr int KQ = NW / 4;                 // workers per tensor-memory lane quarter
  static constexpr int TOKW = kN / KQ;              // epilogue token columns per worker
  static constexpr int NV = NMAT * TOKW;            // accumulator values per worker thread
  static_assert(NSLOT >= 2, "ring too shallow");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(2 * ACC_COLS + (Q4 ? 2 * A_COLS : 0) <= (int)TMEM_COLS, "tensor memory");
};

template <int KIND, int WT, int ACT>
__global__ void __launch_bounds__(RowShape<KIND, WT, ACT>::THREADS, 1) row_gemm_kernel(const __grid_constant__ RowArgs a) {
  using S = RowShape<KIND, WT, ACT>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  TcCtrl &C = *reinterpret_cast<TcCtrl *>(smem + S::CTRL_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  if (tid == 0) ctrl_init<S::NSLOT>(C, S::NW, S::Q4 ? S::NW + 1u : 1u);
  if (warp == 1) tmem_alloc(&C.tmem, S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;
  volatile int *abort_flag = &C.abort_flag;

  pdl_wait();
  pdl_launch_dependents();

  const int T_all = (a.nrows + kM - 1) / kM;
  if (KIND == K_UP) {
    list_tiles(C, a.uwords, a.nwords, T_all);
  } else if (tid == 0) {
    C.n_tiles = T_all;
  }
  if (KIND == K_P1 && a.uwords)  // cleared here, set by pred_s (the next kernel)
    for (int w = cta * S::THREADS + tid; w < a.nwords; w += G * S::THREADS) a.uwords[w] = 0u;
  __syncthreads();
  const long long T = C.n_tiles;
  const long long SK = (a.K + S::STEPK - 1) / S::STEPK;
  const long long W = T * SK;
  // stream-K over min(G, W) CTAs so that every CTA taking part owns a unit
  const int Gs = (int)(W < G ? W : G);
  const Span sp = cta < Gs ? span_of(W, Gs, cta) : Span{0, 0};
  auto tile_of = [&](long long j) -> int { return KIND == K_UP ? C.tlist[j] : (int)j; };

  if (warp == 0) {
    // ------------------------------------------------------------ producer warp
    // A thread issues its bulk copies one after another, so the copies of a
    // unit are spread over the lanes: lane c issues copy c.
    long long i = 0;
    for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      if (i >= S::NSLOT && !mbar_wait_warp(&C.empty[s], ph ^ 1u, abort_flag, a.status)) break;
      const int row0 = tile_of(u / SK) * kM;
      const int k0 = (int)(u % SK) * S::STEPK;
      unsigned char *slot = smem + s * S::SLOTB;
      if (lane == 0) mbar_expect_tx(&C.full[s], S::TX);
      __syncwarp();
      // copies: A boxes (lanes 0..NMAT-1), int4 scale boxes (NMAT..2 NMAT-1), images (next lanes)
      constexpr int LS = S::NMAT, LI = S::Q4 ? 2 * S::NMAT : S::NMAT;
      if (lane < LS) {
        tma_load_2d(su32(slot + lane * S::ABOX), lane == 0 ? &a.tm0 : &a.tm1, S::Q4 ? k0 / 2 : k0, row0, &C.full[s]);
      } else if (S::Q4 && lane < LI) {
        const int mat = lane - LS;
        tma_load_2d(su32(slot + S::SC_OFF + mat * S::SBOX), mat == 0 ? &a.ts0 : &a.ts1, k0 / 16, row0, &C.full[s]);
      } else if (lane < LI + S::NIMG) {
        const int nb = lane - LI;
        const size_t ib = (size_t)(k0 / 16) * kBlk;
        bulk_g2s(su32(slot + S::IMG_OFF + nb * (S::STEPK / 16) * kBlk), (nb == 0 ? a.img0 : a.img1) + ib,
                 (S::STEPK / 16) * kBlk, &C.full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one lane)
    if (lane == 0) {
      long long i = 0;
      int piece = -1;
      for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        const bool first = (u == sp.u0) || (u % SK == 0);
        if (first) {
          ++piece;
          if (piece >= 2 &&
              !mbar_wait(&C.accfree[piece & 1], (unsigned)(((piece >> 1) & 1) ^ 1), abort_flag, a.status))
            break;
        }
        if (!mbar_wait(&C.full[s], ph, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)((piece & 1) * S::ACC_COLS);
        const uint32_t slot = su32(smem + s * S::SLOTB);
        constexpr uint32_t idesc = idesc_f16(kM, kN, 0, 0);
        if constexpr (!S::Q4) {
          // A straight from the swizzled TMA box: 16 K = 32 bytes along the 128-byte rows
#pragma unroll
          for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int mat = 0; mat < S::NMAT; ++mat)
#pragma unroll
              for (int nb = 0; nb < S::NIMG; ++nb) {
                const uint64_t ad = sdesc(slot + mat * S::ABOX + j * 32, 16, 1024, kSw128);
                const uint64_t bd = sdesc(slot + S::IMG_OFF + nb * 4 * kBlk + j * kBlk, 128, 256);
                mma_ss(acc + mat * kN, ad, bd, idesc, (first && j == 0 && nb == 0) ? 0u : 1u);
              }
          mma_commit(&C.empty[s]);
        } else {
          // two 128-K halves, each dequantised by the workers into a tensor-memory A buffer
#pragma unroll 1
          for (int sub = 0; sub < 2; ++sub) {
            const long long ia = 2 * i + sub;
            const int b = (int)(ia & 1);
            if (!mbar_wait(&C.afull[b], (unsigned)((ia >> 1) & 1), abort_flag, a.status)) break;
            tc_fence_after();
            const uint32_t abuf = tmem + (uint32_t)(2 * S::ACC_COLS + b * S::A_COLS);
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
              for (int mat = 0; mat < S::NMAT; ++mat) {
                const uint64_t bd = sdesc(slot + S::IMG_OFF + (sub * 8 + j) * kBlk, 128, 256);
                mma_ts(acc + mat * kN, abuf + mat * 64 + j * 8, bd, idesc, (first && sub == 0 && j == 0) ? 0u : 1u);
              }
            mma_commit(&C.afree[b]);
          }
          if (*abort_flag) break;
          mma_commit(&C.empty[s]);
        }
        const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
        if (last) mma_commit(&C.accfull[piece & 1]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ workers: int4 A operand + epilogues
    const int w = warp - 2;       // 0..NW-1
    const int q = warp & 3;       // tensor-memory lane quarter of this warp
    const int kq = w >> 2;        // slice of a dequant step's K; of the epilogue's tokens
    const int m = q * 32 + lane;  // row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    unsigned wphase = 0;
    bool ok = true;
    long long i = 0;
    int piece = -1;
    long long piece_u0 = sp.u0;
    for (long long u = sp.u0; u < sp.u1 && ok; ++u, ++i) {
      const long long j_tile = u / SK;
      if ((u == sp.u0) || (u % SK == 0)) {
        ++piece;
        piece_u0 = u;
      }
      if constexpr (S::Q4) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        if (!mbar_wait_warp(&C.full[s], ph, abort_flag, a.status)) break;
        const unsigned char *slot = smem + s * S::SLOTB;
        bool fine = true;
#pragma unroll 1
        for (int sub = 0; sub < 2 && fine; ++sub) {
          const long long ia = 2 * i + sub;
          const int b = (int)(ia & 1);
          if (ia >= 2 && !mbar_wait_warp(&C.afree[b], (unsigned)(((ia >> 1) & 1) ^ 1), abort_flag, a.status)) {
            fine = false;
            break;
          }
          // this thread: row m, GPS consecutive 32-element groups of the unit
          // (one 16-byte chunk each), GPS = 4 / KQ
          constexpr int GPS = 4 / S::KQ;
#pragma unroll
          for (int gg = 0; gg < GPS; ++gg) {
            const int g = sub * 4 + kq * GPS + gg;
            const uint32_t acol = lane_base + (uint32_t)(2 * S::ACC_COLS + b * S::A_COLS + (kq * GPS + gg) * 16);
#pragma unroll
            for (int mat = 0; mat < S::NMAT; ++mat) {
              // packed row m of the swizzled box: 16-byte chunk g sits at (g ^ (m % 8)) * 16
              const uint4 pk =
                  *reinterpret_cast<const uint4 *>(slot + mat * S::ABOX + m * 128 + ((g ^ (m & 7)) << 4));
              const __half sc = *reinterpret_cast<const __half *>(slot + S::SC_OFF + mat * S::SBOX + m * 16 + g * 2);
              const __half2 s2 = __halves2half2(sc, sc);
              const uint32_t wds[4] = {pk.x, pk.y, pk.z, pk.w};
              uint32_t v[16];
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                uint32_t o[4];
                q8_to_h4_paired(wds[t], s2, o);
#pragma unroll
                for (int c = 0; c < 4; ++c) v[t * 4 + c] = o[c];
              }
              tmem_st16(acol + mat * 64, v);
            }
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&C.afull[b]);
        }
        if (!fine) break;
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[s]);
      }
      const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
      if (!last) continue;

      // ---------------------------------------------------------- epilogue of one piece
      const int pb = piece & 1;
      if (!mbar_wait_warp(&C.accfull[pb], (unsigned)((piece >> 1) & 1), abort_flag, a.status)) break;
      tc_fence_after();
      float v[S::NV];
#pragma unroll
      for (int mat = 0; mat < S::NMAT; ++mat) {
        const uint32_t col = lane_base + (uint32_t)(pb * S::ACC_COLS + mat * kN + kq * S::TOKW);
        if constexpr (S::TOKW == 16) {
          float t[16];
          tmem_ld16(col, t);
#pragma unroll
          for (int j = 0; j < 16; ++j) v[mat * 16 + j] = t[j];
        } else {
          float t[8];
          tmem_ld8(col, t);
#pragma unroll
          for (int j = 0; j < 8; ++j) v[mat * 8 + j] = t[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.accfree[pb]);

      const bool whole = (piece_u0 % SK == 0) && ((u + 1) % SK == 0);
      if (!whole && !stream_k_finish<S::NV>(v, a.part, a.ctr, (int)j_tile, SK, W, Gs, cta, sp.u0, w, lane, C,
                                            wphase, abort_flag, a.status, &ok))
        continue;

      // ---------------------------------------------------------- finish the tile
      const int row = tile_of(j_tile) * kM + m;  // r index (pred_h) or neuron (pred_s, ffn_up)
      if constexpr (KIND == K_P1) {
        if (row < a.nrows) {
          const size_t boff = (size_t)(row >> 4) * kBlk;
#pragma unroll
          for (int j = 0; j < S::TOKW; ++j) {
            const int n = kq * S::TOKW + j;
            const __half hi = __float2half_rn(v[j]);
            const __half lo = __float2half_rn(v[j] - __half2float(hi));
            const uint32_t o = img_off(n, row & 15);
            *reinterpret_cast<__half *>(a.out0 + boff + o) = hi;
            *reinterpret_cast<__half *>(a.out1 + boff + o) = lo;
          }
        }
      } else if constexpr (KIND == K_P2) {
        const bool valid = row < a.nrows;
        const float bias = valid ? __ldg(a.bias + row) : 0.f;
        const int word = (int)(j_tile * kM + q * 32) >> 5;
        unsigned any = 0u;
#pragma unroll
        for (int j = 0; j < S::TOKW; ++j) {
          const int n = kq * S::TOKW + j;
          const unsigned bits = __ballot_sync(0xffffffffu, valid && (v[j] + bias > 0.f));
          if (lane == 0 && n < a.B && word < a.nwords) {
            a.mask_out[(size_t)n * a.nwords + word] = bits;
            any |= bits;
          }
        }
        if (lane == 0 && any) atomicOr(a.uwords + word, any);  // union words (order-free)
      } else {
        // a image position: listed tile j_tile, row m.  Up to 16 tokens the
        // image holds a_hi = fp16(a) in column n and a_lo = fp16(a - a_hi) in
        // column n + 16 (the down GEMM adds the two), so a keeps about 22
        // bits; above 16 tokens every column is a token and a is fp16(a).
        const bool split = a.B <= kN / 2;
        const bool valid = row < a.nrows;
        const float b1 = (ACT == ACT_RELU && valid) ? __ldg(a.bias + row) : 0.f;
        const long long pos = j_tile * kM + m;
        const size_t boff = (size_t)(pos >> 4) * kBlk;
#pragma unroll
        for (int j = 0; j < S::TOKW; ++j) {
          const int n = kq * S::TOKW + j;
          if (split && n >= kN / 2) continue;  // column of a lo part, written below
          float av = 0.f;
          if (valid && n < a.B) {
            const uint32_t bits = __ldg(a.mask + (size_t)n * a.nwords + (row >> 5));
            if ((bits >> (row & 31)) & 1u) {
              if constexpr (ACT == ACT_RELU) {
                const float pre = v[j] + b1;
                av = pre > 0.f ? pre : 0.f;
              } else {
                av = silu(v[S::TOKW + j]) * v[j];  // silu(gate) * up
              }
            }
          }
          const __half hi = __float2half_rn(av);
          *reinterpret_cast<__half *>(a.out0 + boff + img_off(n, (int)(pos & 15))) = hi;
          if (split)
            *reinterpret_cast<__half *>(a.out0 + boff + img_off(n + kN / 2, (int)(pos & 15))) =
                __float2half_rn(av - __half2float(hi));
        }
      }
    }
  }
  teardown(warp, tmem, S::TMEM_COLS);
}

// ---------------------------------------------------------------- down projection (A in shared memory)
struct DownArgs {
  CUtensorMap tm;               // W2T: fp16 [f x d] (box 64 x 64) or packed int4 bytes [f x d/2] (box 128 x 64)
  CUtensorMap ts;               // int4 scale bytes [f x d/16] (box 16 x 64)
  const uint32_t *uwords;       // union mask words (the same tile list as ffn_up)
  int nwords, f, d, B;
  const unsigned char *aimg;    // a image, K = the listed tiles' neurons
  float *y;                     // [B x d]
  int accumulate;
  float *part;
  int *ctr;
  int *status;
};

template <int WT>
struct DownShape {
  static constexpr bool Q4 = WT == W_INT4;
  // fp16: four 64-column boxes of 64 neurons x 128 B (swizzled, the MMA's
  // MN-major A as is); int4: one 64 x 128 B packed box + a 64 x 16 B scale box
  static constexpr int ABYTES = Q4 ? 8192 : 4 * 8192;
  static constexpr int SBYTES = Q4 ? 1024 : 0;
  static constexpr int IMGB = (kDownStepK / 16) * kBlk;  // 4 KB
  static constexpr int IMG_OFF = ABYTES + SBYTES;
  static constexpr int SLOTB = (IMG_OFF + IMGB + 1023) / 1024 * 1024;
  static constexpr int ABUF = Q4 ? kDownStepK * kDownTileD * 2 : 0;  // int4: dequantised canonical A, 32 KB
  static constexpr int NSLOT_FIT = (kSmemBudget - 2 * ABUF) / SLOTB;
  static constexpr int NSLOT = NSLOT_FIT > kMaxSlots ? kMaxSlots : NSLOT_FIT;
  static constexpr int TX = IMG_OFF + IMGB;
  static constexpr int A_OFF = NSLOT * SLOTB;
  static constexpr int CTRL_OFF = A_OFF + 2 * ABUF;
  static constexpr int SMEM = CTRL_OFF + kCtrlBytes + 1024;
  static constexpr uint32_t TMEM_COLS = 128;  // 2 buffers x 2 M-halves x 32 tokens
  static_assert(NSLOT >= 2, "ring too shallow");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) ffn_down_kernel(const __grid_constant__ DownArgs a) {
  using S = DownShape<WT>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  TcCtrl &C = *reinterpret_cast<TcCtrl *>(smem + S::CTRL_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  if (tid == 0) ctrl_init<S::NSLOT>(C, 8u, S::Q4 ? 9u : 1u);
  if (warp == 1) tmem_alloc(&C.tmem, S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;
  volatile int *abort_flag = &C.abort_flag;

  pdl_wait();
  pdl_launch_dependents();

  list_tiles(C, a.uwords, a.nwords, (a.f + kM - 1) / kM);
  const int d = a.d;
  const long long T = (d + kDownTileD - 1) / kDownTileD;
  const long long SK = (long long)C.n_tiles * (kM / kDownStepK);
  const long long W = T * SK;
  if (W == 0 && !a.accumulate) {
    // no predicted neuron: y = 0
    const int n = a.B * d;
    for (int e = cta * kThreads + tid; e < n; e += G * kThreads) a.y[e] = 0.f;
  }
  const int Gs = (int)(W < G ? W : G);
  const Span sp = cta < Gs ? span_of(W, Gs, cta) : Span{0, 0};

  if (warp == 0) {
    // ------------------------------------------------------------ producer warp (lane c issues copy c)
    long long i = 0;
    for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      if (i >= S::NSLOT && !mbar_wait_warp(&C.empty[s], ph ^ 1u, abort_flag, a.status)) break;
      const int dcol0 = (int)(u / SK) * kDownTileD;
      const long long kstep = u % SK;  // 64-neuron half of listed tile kstep / 2
      const int row0 = C.tlist[kstep >> 1] * kM + (int)(kstep & 1) * kDownStepK;
      unsigned char *slot = smem + s * S::SLOTB;
      if (lane == 0) mbar_expect_tx(&C.full[s], S::TX);
      __syncwarp();
      constexpr int NA = S::Q4 ? 2 : 4;  // int4: packed + scales; fp16: four 64-column boxes
      if (lane < NA) {
        if constexpr (S::Q4) {
          if (lane == 0) tma_load_2d(su32(slot), &a.tm, dcol0 / 2, row0, &C.full[s]);
          else tma_load_2d(su32(slot + S::ABYTES), &a.ts, dcol0 / 16, row0, &C.full[s]);
        } else {
          tma_load_2d(su32(slot + lane * 8192), &a.tm, dcol0 + lane * 64, row0, &C.full[s]);
        }
      } else if (lane == NA) {
        bulk_g2s(su32(slot + S::IMG_OFF), a.aimg + (size_t)kstep * S::IMGB, S::IMGB, &C.full[s]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one lane)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kM, kN, 1, 0);
      long long i = 0;
      int piece = -1;
      for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        const int b = (int)(i & 1);
        const bool first = (u == sp.u0) || (u % SK == 0);
        if (first) {
          ++piece;
          if (piece >= 2 &&
              !mbar_wait(&C.accfree[piece & 1], (unsigned)(((piece >> 1) & 1) ^ 1), abort_flag, a.status))
            break;
        }
        if (!mbar_wait(&C.full[s], ph, abort_flag, a.status)) break;
        if (S::Q4 && !mbar_wait(&C.afull[b], (unsigned)((i >> 1) & 1), abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)((piece & 1) * 64);
        const uint32_t slot = su32(smem + s * S::SLOTB);
        const uint32_t abuf = su32(smem + S::A_OFF + b * S::ABUF);
#pragma unroll
        for (int j = 0; j < kDownStepK / 16; ++j) {
          const uint64_t bd = sdesc(slot + S::IMG_OFF + j * kBlk, 128, 256);
#pragma unroll
          for (int hm = 0; hm < 2; ++hm) {
            uint64_t ad;
            if constexpr (S::Q4) {
              // canonical no-swizzle MN-major: 8-position groups of d 128 B apart, 8-neuron groups 4096 B apart
              ad = sdesc(abuf + (uint32_t)(j * 2 * 4096 + hm * 2048), 4096, 128);
            } else {
              // swizzled boxes: 64-column blocks 8 KB apart, 8-neuron groups 1 KB apart
              ad = sdesc(slot + (uint32_t)(hm * 2 * 8192 + j * 2048), 8192, 1024, kSw128);
            }
            mma_ss(acc + hm * kN, ad, bd, idesc, (first && j == 0) ? 0u : 1u);
          }
        }
        if (S::Q4) mma_commit(&C.afree[b]);
        mma_commit(&C.empty[s]);
        const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
        if (last) mma_commit(&C.accfull[piece & 1]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ workers
    const int w = warp - 2, q = warp & 3, hm = w >> 2;
    const int wt = w * 32 + lane;  // 0..255
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    unsigned wphase = 0;
    bool ok = true;
    long long i = 0;
    int piece = -1;
    long long piece_u0 = sp.u0;
    for (long long u = sp.u0; u < sp.u1 && ok; ++u, ++i) {
      const long long tile = u / SK;
      if ((u == sp.u0) || (u % SK == 0)) {
        ++piece;
        piece_u0 = u;
      }
      if constexpr (S::Q4) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        const int b = (int)(i & 1);
        if (!mbar_wait_warp(&C.full[s], ph, abort_flag, a.status)) break;
        if (i >= 2 && !mbar_wait_warp(&C.afree[b], (unsigned)(((i >> 1) & 1) ^ 1), abort_flag, a.status)) break;
        const unsigned char *slot = smem + s * S::SLOTB;
        unsigned char *ab = smem + S::A_OFF + b * S::ABUF;
        // item (neuron k, group g of 32 d): packed chunk g of row k sits at (g ^ (k % 8)) * 16 in the
        // swizzled box; canonical MN-major A element (d m, neuron k) at
        // (k/8)*4096 + (m/8)*128 + (k%8)*16 + (m%8)*2.  A warp's 32 items take 8
        // consecutive k so its 16-byte stores spread over all banks.
#pragma unroll
        for (int it = wt; it < kDownStepK * 8; it += kThreads - 64) {
          const int k = ((it >> 6) << 3) | (it & 7), g = (it >> 3) & 7;
          const uint4 pk = *reinterpret_cast<const uint4 *>(slot + k * 128 + ((g ^ (k & 7)) << 4));
          const __half sc = *reinterpret_cast<const __half *>(slot + S::ABYTES + k * 16 + g * 2);
          const __half2 s2 = __halves2half2(sc, sc);
          const uint32_t wds[4] = {pk.x, pk.y, pk.z, pk.w};
          unsigned char *dst = ab + (k >> 3) * 4096 + (k & 7) * 16 + g * 4 * 128;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            uint32_t o[4];
            q8_to_h4(wds[t], s2, o);
            *reinterpret_cast<uint4 *>(dst + t * 128) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
        proxy_fence_async();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&C.afull[b]);
          mbar_arrive(&C.empty[s]);
        }
      }
      const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
      if (!last) continue;

      // ---------------------------------------------------------- epilogue
      const int pb = piece & 1;
      if (!mbar_wait_warp(&C.accfull[pb], (unsigned)((piece >> 1) & 1), abort_flag, a.status)) break;
      tc_fence_after();
      float v[32];
      {
        float t0[16], t1[16];
        tmem_ld16(lane_base + (uint32_t)(pb * 64 + hm * kN), t0);
        tmem_ld16(lane_base + (uint32_t)(pb * 64 + hm * kN + 16), t1);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          v[j] = t0[j];
          v[16 + j] = t1[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.accfree[pb]);

      const bool whole = (piece_u0 % SK == 0) && ((u + 1) % SK == 0);
      if (!whole && !stream_k_finish<32>(v, a.part, a.ctr, (int)tile, SK, W, Gs, cta, sp.u0, w, lane, C, wphase,
                                         abort_flag, a.status, &ok))
        continue;
      const int dpos = (int)tile * kDownTileD + hm * kM + q * 32 + lane;
      const bool split = a.B <= kN / 2;  // columns n + 16 hold the a_lo parts
      if (dpos < d) {
#pragma unroll
        for (int n = 0; n < kN; ++n) {
          if (n < a.B) {
            const float yv = split ? v[n] + v[(n + kN / 2) % kN] : v[n];
            float *yp = a.y + (size_t)n * d + dpos;
            *yp = a.accumulate ? *yp + yv : yv;
          }
        }
      }
    }
  }
  teardown(warp, tmem, S::TMEM_COLS);
}

}  // namespace tc
}  // namespace pi
