// pi_tc.cuh -- tensor-core (tcgen05) path for token batches of 16..32.
//
// At batch >= 16 the union of the tokens' predicted sets covers nearly every
// neuron, so each gathered block is a dense contraction (the 16..32 token
// columns are the MMA's N).  Four persistent kernels run it, each on one CTA
// per SM with a stream-K split of its (tile, K-step) work so that all SMs end
// together:
//
//   pred_h  : h^T[r x N]  = P1 u^T              (A = P1 rows, K = d)
//   pred_s  : s^T[f x N]  = P2 (h_hi + h_lo)^T  (A = P2 rows, K = r) + bias,
//             thresholded to the per-token mask words
//   ffn_up  : a^T[U x N]  = act(W_up/gate[union] u^T), zero where the token
//             did not predict the neuron        (A = gathered rows, K = d)
//   ffn_down: y^T[d x N]  = W2T[union]^T a^T    (A = gathered W2T rows, MN-major)
//
// The three "row" kernels use one template (ts_gemm_kernel): a producer warp
// copies 128 rows x 128 K of row data into a shared-memory ring with
// cp.async; eight worker warps move it (dequantising int4) into tensor memory
// as the MMA's A operand; one thread issues tcgen05.mma with the token image
// (B operand) in shared memory; the worker warps also run the epilogue.  The
// down kernel keeps A in shared memory (the d positions are the MMA's M, so a
// neuron row lands as 16-byte MN-major pieces).
//
// Token operands are stored as "images": per 16-deep K block, 1 KB holding
// the 32 token rows in the canonical no-swizzle K-major UMMA layout (core
// matrices of 8 tokens x 8 K, 16-byte rows).  Padding tokens and K beyond the
// row length are zero, so padded MMA work adds exact zeros.
//
// Stream-K: a kernel's W = tiles x steps units are split into G contiguous
// spans.  A tile whose steps span several CTAs is finished by the last CTA to
// arrive (per-tile counter): it adds the pieces' fp32 partials in K order, so
// the result does not depend on timing.  Counters reset themselves.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "pi_device.cuh"

namespace pi {
namespace tc {

constexpr int kN = 32;        // MMA N: token columns (batches of 16..32 are zero-padded)
constexpr int kM = 128;       // MMA M: rows of a tile
constexpr int kStepK = 128;   // K per pipeline step of the row kernels
constexpr int kBlk = 1024;    // bytes of one 16-deep K block of a token image
constexpr int kStepImg = 8 * kBlk;
constexpr int kThreads = 320; // warp 0 producer, warp 1 MMA issuer, warps 2..9 workers
constexpr int kWorkerThreads = 256;
constexpr int kSmemBudget = 212 * 1024;
constexpr int kPartFloats = 128 * 64;  // largest per-piece partial (floats)
constexpr int kDownTileD = 256;        // d positions per down-projection tile (two M=128 MMAs)
constexpr int kDownStepK = 64;         // union positions per down-projection step
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
PI_DEV bool mbar_test(uint64_t *b, unsigned parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(su32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity.  Gives up when another
// role of the CTA has aborted or after kWaitNs (recording a timeout).
__device__ __noinline__ bool mbar_wait_slow(uint64_t *b, unsigned parity, volatile int *abort_flag, int *status) {
  const unsigned long long t0 = now_ns();
  for (;;) {
    if (mbar_test(b, parity)) return true;
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

// 16-byte cp.async; src_bytes 0 fills the destination with zeros
PI_DEV void cp16(uint32_t dst, const void *src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// arrive on b once all earlier cp.async of this thread have landed
PI_DEV void cp_arrive(uint64_t *b) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(su32(b)) : "memory");
}
PI_DEV void cp_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

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

// UMMA shared-memory descriptor, no swizzle: start, leading and stride byte offsets
PI_DEV uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
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

// ---------------------------------------------------------------- stream-K
struct Span {
  long long u0, u1;  // this CTA's units [u0, u1)
};
PI_DEV Span span_of(long long W, int G, int c) { return Span{W * c / G, W * (c + 1) / G}; }
// CTA owning unit u
PI_DEV int owner_of(long long u, long long W, int G) { return (int)(((u + 1) * G + W - 1) / W) - 1; }

// ---------------------------------------------------------------- token image
// u [B x d] fp16 -> image of ceil(d/128)*8 blocks; tokens >= B and k >= d are 0
__global__ void __launch_bounds__(256) u_image_kernel(const __half *__restrict__ u, int B, int d,
                                                      unsigned char *__restrict__ img) {
  pdl_wait();
  pdl_launch_dependents();
  const int nblk = (d + kStepK - 1) / kStepK * 8;
  const int per_tok = nblk * 2;  // 16-byte pieces per token row of the image
  const int total = kN * per_tok;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < total; c += gridDim.x * blockDim.x) {
    const int n = c / per_tok, j = c - n * per_tok;
    const int blk = j >> 1, kh = j & 1;
    const int k0 = blk * 16 + kh * 8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (n < B && k0 < d) v = *reinterpret_cast<const uint4 *>(u + (size_t)n * d + k0);
    *reinterpret_cast<uint4 *>(img + (size_t)blk * kBlk + img_off(n, kh * 8)) = v;
  }
}

// ---------------------------------------------------------------- row GEMM (A in tensor memory)
struct TsArgs {
  const void *w0, *w1;           // row data of matrix 0 / 1 ([rows x K] fp16, or packed int4)
  const __half *s0, *s1;         // int4 group scales [rows x K/32]
  const int32_t *rowlist;        // ffn_up: union position -> neuron id
  const int32_t *rowcount;       // ffn_up: device union size U
  int nrows;                     // number of rows when rowcount is null
  int K;                         // row length (elements)
  const unsigned char *img0;     // B operand image (u, or h_hi)
  const unsigned char *img1;     // pred_s: h_lo image
  const float *bias;             // pred_s: predictor bias; ffn_up ReLU: b_up
  const uint32_t *mask;          // ffn_up: per-token mask words [B x nwords]
  uint32_t *mask_out;            // pred_s: per-token mask words [B x nwords]
  int nwords, B;
  unsigned char *out0, *out1;    // pred_h: h_hi / h_lo images; ffn_up: a image
  float *part;                   // stream-K partials [G x 2 x kPartFloats]
  int *ctr;                      // per-tile arrival counters (zero between launches)
  int *status;
};

struct TsCtrl {
  uint64_t full[6], img_full[6], empty[6], img_empty[6];
  uint64_t afull[2], afree[2], accfull[2], accfree[2];
  uint64_t wbar;  // the 256 worker threads' barrier (stream-K fix-up)
  uint32_t tmem;
  int abort_flag;
  int is_last;
  int rows[kM];   // producer: row ids of the current tile / step (-1: padding)
};
constexpr int kCtrlBytes = 1024;
static_assert(sizeof(TsCtrl) <= kCtrlBytes, "control block");

template <int KIND, int WT, int ACT>
struct TsShape {
  static constexpr int NMAT = (KIND == K_UP && ACT == ACT_SWIGLU) ? 2 : 1;
  static constexpr int NIMG = KIND == K_P2 ? 2 : 1;
  static constexpr bool Q4 = WT == W_INT4;
  // staging row pitch per matrix for one step: int4 64 B packed + 16 B scales,
  // fp16 256 B + 16 B pad (the pad spreads rows over the banks)
  static constexpr int ROWB = Q4 ? 80 : 272;
  static constexpr int SLOTB = NMAT * kM * ROWB;
  static constexpr int IMGB = NIMG * kStepImg;
  static constexpr int NSLOT_FIT = kSmemBudget / (SLOTB + IMGB);
  static constexpr int NSLOT = NSLOT_FIT > 6 ? 6 : NSLOT_FIT;
  static constexpr int IMG_OFF = 0;
  static constexpr int STAGE_OFF = NSLOT * IMGB;
  static constexpr int CTRL_OFF = STAGE_OFF + NSLOT * SLOTB;
  static constexpr int SMEM = CTRL_OFF + kCtrlBytes;
  static constexpr int ACC_COLS = NMAT * kN;  // per accumulator buffer
  static constexpr int A_COLS = NMAT * 64;    // per A buffer (128 K of fp16 pairs)
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(NSLOT >= 2, "ring too shallow");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(2 * ACC_COLS + 2 * A_COLS <= (int)TMEM_COLS, "tensor memory");
};


template <int NSLOT>
PI_DEV void ctrl_init(TsCtrl &C) {
  for (int s = 0; s < NSLOT; ++s) {
    mbar_init(&C.full[s], 32);      // the producer warp's cp.async arrivals
    mbar_init(&C.img_full[s], 1);   // expect_tx of the image bulk copy
    mbar_init(&C.empty[s], 8);      // the 8 worker warps
    mbar_init(&C.img_empty[s], 1);  // MMA commit
  }
  for (int b = 0; b < 2; ++b) {
    mbar_init(&C.afull[b], 8);
    mbar_init(&C.afree[b], 1);
    mbar_init(&C.accfull[b], 1);
    mbar_init(&C.accfree[b], 8);
  }
  mbar_init(&C.wbar, kWorkerThreads);
  C.abort_flag = 0;
  C.is_last = 0;
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Stream-K fix-up for one worker thread's NV accumulator values of a piece
// that does not cover its whole tile (G: the CTAs the units were split
// over).  Publishes the piece; the CTA whose
// piece arrives last sums all pieces in K order into v and returns true.
// *ok turns false when a bounded wait gave up.
template <int NV>
PI_DEV bool stream_k_finish(float (&v)[NV], float *part, int *ctr, int tile, long long SK, long long W, int G,
                            int cta, long long u0, int w, int lane, TsCtrl &C, unsigned &wphase,
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
  float acc[NV];
#pragma unroll
  for (int j = 0; j < NV; ++j) acc[j] = 0.f;
  for (int c = c0; c <= c1; ++c) {
    if (c == cta) {
#pragma unroll
      for (int j = 0; j < NV; ++j) acc[j] += v[j];
    } else {
      const int cslot = (int)(span_of(W, G, c).u0 / SK) == tile ? 0 : 1;
      const float *pp = part + ((size_t)c * 2 + cslot) * kPartFloats;
#pragma unroll
      for (int j = 0; j < NV; ++j) acc[j] += __ldcg(pp + (w * NV + j) * 32 + lane);
    }
  }
#pragma unroll
  for (int j = 0; j < NV; ++j) v[j] = acc[j];
  return true;
}

// Waits for the issuer's last commit (all MMAs done), then releases tensor memory.
PI_DEV void teardown(TsCtrl &C, const Span &sp, int warp, int lane, uint32_t tmem, uint32_t ncols,
                     volatile int *abort_flag, int *status) {
  if (warp == 1 && lane == 0) {
    const long long n_steps = sp.u1 - sp.u0;
    if (n_steps > 0 && !*abort_flag) {
      const long long il = n_steps - 1;
      mbar_wait(&C.afree[il & 1], (unsigned)((il >> 1) & 1), abort_flag, status);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, ncols);
}

template <int KIND, int WT, int ACT>
__global__ void __launch_bounds__(kThreads, 1) ts_gemm_kernel(const TsArgs a) {
  using S = TsShape<KIND, WT, ACT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  TsCtrl &C = *reinterpret_cast<TsCtrl *>(smem + S::CTRL_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  if (tid == 0) ctrl_init<S::NSLOT>(C);
  if (warp == 1) tmem_alloc(&C.tmem, S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;
  volatile int *abort_flag = &C.abort_flag;

  pdl_wait();
  pdl_launch_dependents();

  const int nrows = a.rowcount ? *a.rowcount : a.nrows;
  const long long T = (nrows + kM - 1) / kM;
  const long long SK = (a.K + kStepK - 1) / kStepK;
  const long long W = T * SK;
  // stream-K over min(G, W) CTAs so that every CTA taking part owns a unit
  const int Gs = (int)(W < G ? W : G);
  const Span sp = cta < Gs ? span_of(W, Gs, cta) : Span{0, 0};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const size_t rowB = S::Q4 ? (size_t)a.K / 2 : (size_t)a.K * 2;
    const size_t srowB = (size_t)a.K / 16;  // int4 scale bytes per row
    long long cur_tile = -1;
    long long i = 0;
    for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      if (i >= S::NSLOT) {
        if (!mbar_wait_warp(&C.empty[s], ph ^ 1u, abort_flag, a.status)) break;
        if (!mbar_wait_warp(&C.img_empty[s], ph ^ 1u, abort_flag, a.status)) break;
      }
      const long long tile = u / SK;
      const int step = (int)(u % SK);
      if (tile != cur_tile) {
        cur_tile = tile;
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const long long p = tile * kM + lane + 32 * j;
          C.rows[lane + 32 * j] = p < nrows ? (a.rowlist ? __ldg(a.rowlist + p) : (int)p) : -1;
        }
        __syncwarp();
      }
      if (lane == 0) {
        mbar_expect_tx(&C.img_full[s], S::IMGB);
        const uint32_t d0 = su32(smem + S::IMG_OFF + s * S::IMGB);
        bulk_g2s(d0, a.img0 + (size_t)step * kStepImg, kStepImg, &C.img_full[s]);
        if (S::NIMG == 2) bulk_g2s(d0 + kStepImg, a.img1 + (size_t)step * kStepImg, kStepImg, &C.img_full[s]);
      }
      // rows as 16-byte pieces, zero-filled beyond the row and for padding rows
      const uint32_t st0 = su32(smem + S::STAGE_OFF + s * S::SLOTB);
      const int k0 = step * kStepK;
#pragma unroll
      for (int mat = 0; mat < S::NMAT; ++mat) {
        const unsigned char *wb = reinterpret_cast<const unsigned char *>(mat == 0 ? a.w0 : a.w1);
        const uint32_t sm0 = st0 + mat * kM * S::ROWB;
        if constexpr (S::Q4) {
          // 5 pieces per row: 4 x 16 B of packed nibbles (128 elements) and
          // the 16-byte block of the 8 group scales of the enclosing 256 elements
          const unsigned char *sb = reinterpret_cast<const unsigned char *>(mat == 0 ? a.s0 : a.s1);
#pragma unroll 4
          for (int qq = lane; qq < kM * 5; qq += 32) {
            const int m = qq / 5, c = qq - m * 5;
            const int rid = C.rows[m];
            const uint32_t dst = sm0 + m * S::ROWB + c * 16;
            if (c < 4) {
              const bool ok = rid >= 0 && k0 + c * 32 < a.K;
              cp16(dst, wb + (ok ? (size_t)rid * rowB + (size_t)k0 / 2 + c * 16 : 0), ok ? 16u : 0u);
            } else {
              const bool ok = rid >= 0;
              cp16(dst, sb + (ok ? (size_t)rid * srowB + (size_t)(k0 / 256) * 16 : 0), ok ? 16u : 0u);
            }
          }
        } else {
#pragma unroll 4
          for (int qq = lane; qq < kM * 16; qq += 32) {
            const int m = qq >> 4, c = qq & 15;
            const int rid = C.rows[m];
            const bool ok = rid >= 0 && k0 + c * 8 < a.K;
            cp16(sm0 + m * S::ROWB + c * 16, wb + (ok ? (size_t)rid * rowB + (size_t)(k0 + c * 8) * 2 : 0),
                 ok ? 16u : 0u);
          }
        }
      }
      cp_arrive(&C.full[s]);
    }
    cp_wait_all();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kM, kN, 0, 0);
      long long i = 0;
      int piece = -1;
      for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        const int b = (int)(i & 1);
        const unsigned bph = (unsigned)((i >> 1) & 1);
        const bool first = (u == sp.u0) || (u % SK == 0);
        if (first) {
          ++piece;
          if (piece >= 2 &&
              !mbar_wait(&C.accfree[piece & 1], (unsigned)(((piece >> 1) & 1) ^ 1), abort_flag, a.status))
            break;
        }
        if (!mbar_wait(&C.afull[b], bph, abort_flag, a.status)) break;
        if (!mbar_wait(&C.img_full[s], ph, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)((piece & 1) * S::ACC_COLS);
        const uint32_t abuf = tmem + (uint32_t)(2 * S::ACC_COLS + b * S::A_COLS);
        const uint32_t img = su32(smem + S::IMG_OFF + s * S::IMGB);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
#pragma unroll
          for (int mat = 0; mat < S::NMAT; ++mat) {
#pragma unroll
            for (int nb = 0; nb < S::NIMG; ++nb) {
              const uint64_t bd = sdesc(img + nb * kStepImg + j * kBlk, 128, 256);
              const uint32_t accum = (first && j == 0 && nb == 0) ? 0u : 1u;
              mma_ts(acc + mat * kN, abuf + mat * 64 + j * 8, bd, idesc, accum);
            }
          }
        }
        mma_commit(&C.afree[b]);
        mma_commit(&C.img_empty[s]);
        const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
        if (last) mma_commit(&C.accfull[piece & 1]);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ workers: A operand + epilogue
    const int w = warp - 2;       // 0..7
    const int q = warp & 3;       // tensor-memory lane quarter of this warp
    const int h = w >> 2;         // K half of a step; token half of the epilogue
    const int m = q * 32 + lane;  // row within the tile
    const uint32_t lane_base = tmem + ((uint32_t)(q * 32) << 16);
    unsigned wphase = 0;
    bool ok = true;
    long long i = 0;
    int piece = -1;
    long long piece_u0 = sp.u0;
    for (long long u = sp.u0; u < sp.u1 && ok; ++u, ++i) {
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      const int b = (int)(i & 1);
      const unsigned bph = (unsigned)((i >> 1) & 1);
      const long long tile = u / SK;
      const int step = (int)(u % SK);
      if ((u == sp.u0) || (step == 0)) {
        ++piece;
        piece_u0 = u;
      }
      if (!mbar_wait_warp(&C.full[s], ph, abort_flag, a.status)) break;
      if (i >= 2 && !mbar_wait_warp(&C.afree[b], bph ^ 1u, abort_flag, a.status)) break;
      const unsigned char *st = smem + S::STAGE_OFF + s * S::SLOTB;
      const uint32_t acol = lane_base + (uint32_t)(2 * S::ACC_COLS + b * S::A_COLS + h * 32);
#pragma unroll
      for (int mat = 0; mat < S::NMAT; ++mat) {
        const unsigned char *row = st + mat * kM * S::ROWB + m * S::ROWB;
        uint32_t v[32];
        if constexpr (S::Q4) {
          const uint4 p0 = *reinterpret_cast<const uint4 *>(row + h * 32);
          const uint4 p1 = *reinterpret_cast<const uint4 *>(row + h * 32 + 16);
          const uint32_t sc = *reinterpret_cast<const uint32_t *>(row + 64 + ((step & 1) * 4 + h * 2) * 2);
          const __half s_lo = __ushort_as_half((unsigned short)(sc & 0xFFFFu));
          const __half s_hi = __ushort_as_half((unsigned short)(sc >> 16));
          const __half2 sA = __halves2half2(s_lo, s_lo), sB = __halves2half2(s_hi, s_hi);
          const uint32_t wds[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            uint32_t o[4];
            q8_to_h4(wds[t], t < 4 ? sA : sB, o);
#pragma unroll
            for (int c = 0; c < 4; ++c) v[t * 4 + c] = o[c];
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint4 p = *reinterpret_cast<const uint4 *>(row + h * 128 + t * 16);
            v[t * 4 + 0] = p.x;
            v[t * 4 + 1] = p.y;
            v[t * 4 + 2] = p.z;
            v[t * 4 + 3] = p.w;
          }
        }
        tmem_st32(acol + mat * 64, v);
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&C.afull[b]);
        mbar_arrive(&C.empty[s]);
      }
      const bool last = (u + 1 == sp.u1) || ((u + 1) % SK == 0);
      if (!last) continue;

      // ---------------------------------------------------------- epilogue of one piece
      const int pb = piece & 1;
      if (!mbar_wait_warp(&C.accfull[pb], (unsigned)((piece >> 1) & 1), abort_flag, a.status)) break;
      tc_fence_after();
      float v[S::NMAT * 16];
#pragma unroll
      for (int mat = 0; mat < S::NMAT; ++mat) {
        float t[16];
        tmem_ld16(lane_base + (uint32_t)(pb * S::ACC_COLS + mat * kN + h * 16), t);
#pragma unroll
        for (int j = 0; j < 16; ++j) v[mat * 16 + j] = t[j];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.accfree[pb]);

      const bool whole = (piece_u0 % SK == 0) && ((u + 1) % SK == 0);
      if (!whole && !stream_k_finish<S::NMAT * 16>(v, a.part, a.ctr, (int)tile, SK, W, Gs, cta, sp.u0, w, lane, C,
                                                   wphase, abort_flag, a.status, &ok))
        continue;

      // ---------------------------------------------------------- finish the tile
      const int row = (int)(tile * kM) + m;  // r index (pred_h), neuron (pred_s), union position (ffn_up)
      if constexpr (KIND == K_P1) {
        if (row < nrows) {
          const size_t boff = (size_t)(row >> 4) * kBlk;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = h * 16 + j;
            const __half hi = __float2half_rn(v[j]);
            const __half lo = __float2half_rn(v[j] - __half2float(hi));
            const uint32_t o = img_off(n, row & 15);
            *reinterpret_cast<__half *>(a.out0 + boff + o) = hi;
            *reinterpret_cast<__half *>(a.out1 + boff + o) = lo;
          }
        }
      } else if constexpr (KIND == K_P2) {
        const bool valid = row < nrows;
        const float bias = valid ? __ldg(a.bias + row) : 0.f;
        const int word = (int)(tile * kM + q * 32) >> 5;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = h * 16 + j;
          const unsigned bits = __ballot_sync(0xffffffffu, valid && (v[j] + bias > 0.f));
          if (lane == 0 && n < a.B && word < a.nwords) a.mask_out[(size_t)n * a.nwords + word] = bits;
        }
      } else {
        const bool valid = row < nrows;
        const int neuron = valid ? __ldg(a.rowlist + row) : 0;
        const float b1 = (ACT == ACT_RELU && valid) ? __ldg(a.bias + neuron) : 0.f;
        const size_t boff = (size_t)(row >> 4) * kBlk;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = h * 16 + j;
          float av = 0.f;
          if (valid && n < a.B) {
            const uint32_t bits = __ldg(a.mask + (size_t)n * a.nwords + (neuron >> 5));
            if ((bits >> (neuron & 31)) & 1u) {
              if constexpr (ACT == ACT_RELU) {
                const float pre = v[j] + b1;
                av = pre > 0.f ? pre : 0.f;
              } else {
                av = silu(v[16 + j]) * v[j];  // silu(gate) * up
              }
            }
          }
          *reinterpret_cast<__half *>(a.out0 + boff + img_off(n, row & 15)) = __float2half_rn(av);
        }
      }
    }
  }
  teardown(C, sp, warp, lane, tmem, S::TMEM_COLS, abort_flag, a.status);
}

// ---------------------------------------------------------------- down projection (A in shared memory)
struct DownArgs {
  const void *w;                 // W2T rows [f x d] fp16, or packed int4 [f x d/2]
  const __half *s;               // int4 scales [f x d/32]
  const int32_t *rowlist;        // union position -> neuron
  const int32_t *rowcount;       // U
  int d, B;
  const unsigned char *aimg;     // a image (union positions as K)
  float *y;                      // [B x d]
  int accumulate;
  float *part;
  int *ctr;
  int *status;
};

template <int WT>
struct DownShape {
  static constexpr bool Q4 = WT == W_INT4;
  // staging row pitch per union position: int4 128 B packed + 16 B scales; fp16 512 B + 16 pad
  static constexpr int ROWB = Q4 ? 144 : 528;
  static constexpr int SLOTB = kDownStepK * ROWB;
  static constexpr int IMGB = (kDownStepK / 16) * kBlk;  // 4 KB
  static constexpr int ABUF = kDownStepK * kDownTileD * 2;  // 32 KB canonical A per step
  static constexpr int NSLOT_FIT = (kSmemBudget - 2 * ABUF) / (SLOTB + IMGB);
  static constexpr int NSLOT = NSLOT_FIT > 6 ? 6 : NSLOT_FIT;
  static constexpr int A_OFF = 0;
  static constexpr int IMG_OFF = 2 * ABUF;
  static constexpr int STAGE_OFF = IMG_OFF + NSLOT * IMGB;
  static constexpr int CTRL_OFF = STAGE_OFF + NSLOT * SLOTB;
  static constexpr int SMEM = CTRL_OFF + kCtrlBytes;
  static constexpr uint32_t TMEM_COLS = 128;  // 2 buffers x 2 M-halves x 32 tokens
  static_assert(NSLOT >= 2, "ring too shallow");
  static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int WT>
__global__ void __launch_bounds__(kThreads, 1) ffn_down_kernel(const DownArgs a) {
  using S = DownShape<WT>;
  extern __shared__ __align__(1024) unsigned char smem[];
  TsCtrl &C = *reinterpret_cast<TsCtrl *>(smem + S::CTRL_OFF);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, cta = blockIdx.x;

  if (tid == 0) ctrl_init<S::NSLOT>(C);
  if (warp == 1) tmem_alloc(&C.tmem, S::TMEM_COLS);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;
  volatile int *abort_flag = &C.abort_flag;

  pdl_wait();
  pdl_launch_dependents();

  const int U = *a.rowcount;
  const int d = a.d;
  const long long T = (d + kDownTileD - 1) / kDownTileD;
  const long long SK = (U + kDownStepK - 1) / kDownStepK;
  const long long W = T * SK;
  if (W == 0 && !a.accumulate) {
    // empty union: y = 0
    const int n = a.B * d;
    for (int e = cta * kThreads + tid; e < n; e += G * kThreads) a.y[e] = 0.f;
  }
  const int Gs = (int)(W < G ? W : G);
  const Span sp = cta < Gs ? span_of(W, Gs, cta) : Span{0, 0};

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const size_t rowB = S::Q4 ? (size_t)d / 2 : (size_t)d * 2;
    const size_t srowB = (size_t)d / 16;
    const unsigned char *wb = reinterpret_cast<const unsigned char *>(a.w);
    long long i = 0;
    for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      if (i >= S::NSLOT) {
        if (!mbar_wait_warp(&C.empty[s], ph ^ 1u, abort_flag, a.status)) break;
        if (!mbar_wait_warp(&C.img_empty[s], ph ^ 1u, abort_flag, a.status)) break;
      }
      const long long tile = u / SK, step = u % SK;
      const int dcol0 = (int)tile * kDownTileD;
      __syncwarp();
#pragma unroll
      for (int j = 0; j < kDownStepK / 32; ++j) {
        const long long p = step * kDownStepK + lane + 32 * j;
        C.rows[lane + 32 * j] = p < U ? __ldg(a.rowlist + p) : -1;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&C.img_full[s], S::IMGB);
        bulk_g2s(su32(smem + S::IMG_OFF + s * S::IMGB), a.aimg + (size_t)step * S::IMGB, S::IMGB, &C.img_full[s]);
      }
      const uint32_t st0 = su32(smem + S::STAGE_OFF + s * S::SLOTB);
      if constexpr (S::Q4) {
        const unsigned char *sb = reinterpret_cast<const unsigned char *>(a.s);
        // 9 pieces per position: 8 x 16 B packed (256 d) + 16 B of the 8 group scales
#pragma unroll 2
        for (int qq = lane; qq < kDownStepK * 9; qq += 32) {
          const int k = qq / 9, c = qq - k * 9;
          const int rid = C.rows[k];
          const uint32_t dst = st0 + k * S::ROWB + c * 16;
          if (c < 8) {
            const bool ok = rid >= 0 && dcol0 + c * 32 < d;
            cp16(dst, wb + (ok ? (size_t)rid * rowB + (size_t)dcol0 / 2 + c * 16 : 0), ok ? 16u : 0u);
          } else {
            const bool ok = rid >= 0;
            cp16(dst, sb + (ok ? (size_t)rid * srowB + (size_t)dcol0 / 16 : 0), ok ? 16u : 0u);
          }
        }
      } else {
#pragma unroll 4
        for (int qq = lane; qq < kDownStepK * 32; qq += 32) {
          const int k = qq >> 5, c = qq & 31;
          const int rid = C.rows[k];
          const bool ok = rid >= 0 && dcol0 + c * 8 < d;
          cp16(st0 + k * S::ROWB + c * 16, wb + (ok ? (size_t)rid * rowB + (size_t)(dcol0 + c * 8) * 2 : 0),
               ok ? 16u : 0u);
        }
      }
      cp_arrive(&C.full[s]);
    }
    cp_wait_all();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(kM, kN, 1, 0);
      long long i = 0;
      int piece = -1;
      for (long long u = sp.u0; u < sp.u1; ++u, ++i) {
        const int s = (int)(i % S::NSLOT);
        const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
        const int b = (int)(i & 1);
        const unsigned bph = (unsigned)((i >> 1) & 1);
        const bool first = (u == sp.u0) || (u % SK == 0);
        if (first) {
          ++piece;
          if (piece >= 2 &&
              !mbar_wait(&C.accfree[piece & 1], (unsigned)(((piece >> 1) & 1) ^ 1), abort_flag, a.status))
            break;
        }
        if (!mbar_wait(&C.afull[b], bph, abort_flag, a.status)) break;
        if (!mbar_wait(&C.img_full[s], ph, abort_flag, a.status)) break;
        tc_fence_after();
        const uint32_t acc = tmem + (uint32_t)((piece & 1) * 64);
        const uint32_t abase = su32(smem + S::A_OFF + b * S::ABUF);
        const uint32_t img = su32(smem + S::IMG_OFF + s * S::IMGB);
#pragma unroll
        for (int j = 0; j < kDownStepK / 16; ++j) {
          const uint64_t bd = sdesc(img + j * kBlk, 128, 256);
#pragma unroll
          for (int hm = 0; hm < 2; ++hm) {
            // MN-major A: 8-position groups of d 128 B apart, 8-deep K groups 4096 B apart
            const uint64_t ad = sdesc(abase + (uint32_t)(j * 2 * 4096 + hm * 2048), 4096, 128);
            mma_ss(acc + hm * kN, ad, bd, idesc, (first && j == 0) ? 0u : 1u);
          }
        }
        mma_commit(&C.afree[b]);
        mma_commit(&C.img_empty[s]);
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
      const int s = (int)(i % S::NSLOT);
      const unsigned ph = (unsigned)((i / S::NSLOT) & 1);
      const int b = (int)(i & 1);
      const unsigned bph = (unsigned)((i >> 1) & 1);
      const long long tile = u / SK, step = u % SK;
      if ((u == sp.u0) || (step == 0)) {
        ++piece;
        piece_u0 = u;
      }
      if (!mbar_wait_warp(&C.full[s], ph, abort_flag, a.status)) break;
      if (i >= 2 && !mbar_wait_warp(&C.afree[b], bph ^ 1u, abort_flag, a.status)) break;
      const unsigned char *st = smem + S::STAGE_OFF + s * S::SLOTB;
      unsigned char *ab = smem + S::A_OFF + b * S::ABUF;
      // canonical MN-major A: (d position m, union position k) at
      // (k/8)*4096 + (m/8)*128 + (k%8)*16 + (m%8)*2.  A warp's 32 items take
      // 8 consecutive k (the low bits of the item) so its 16-byte stores and
      // loads spread over all banks.
      if constexpr (S::Q4) {
#pragma unroll
        for (int it = wt; it < kDownStepK * 8; it += kWorkerThreads) {
          const int k = ((it >> 6) << 3) | (it & 7), g = (it >> 3) & 7;
          const unsigned char *row = st + k * S::ROWB;
          const uint4 pk = *reinterpret_cast<const uint4 *>(row + g * 16);
          const __half sc = *reinterpret_cast<const __half *>(row + 128 + g * 2);
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
      } else {
#pragma unroll 4
        for (int it = wt; it < kDownStepK * 32; it += kWorkerThreads) {
          const int k = ((it >> 8) << 3) | (it & 7), c = (it >> 3) & 31;
          const uint4 p = *reinterpret_cast<const uint4 *>(st + k * S::ROWB + c * 16);
          *reinterpret_cast<uint4 *>(ab + (k >> 3) * 4096 + c * 128 + (k & 7) * 16) = p;
        }
      }
      proxy_fence_async();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&C.afull[b]);
        mbar_arrive(&C.empty[s]);
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
      if (dpos < d) {
        for (int n = 0; n < a.B; ++n) {
          float *yp = a.y + (size_t)n * d + dpos;
          *yp = a.accumulate ? *yp + v[n] : v[n];
        }
      }
    }
  }
  teardown(C, sp, warp, lane, tmem, S::TMEM_COLS, abort_flag, a.status);
}

}  // namespace tc
}  // namespace pi
