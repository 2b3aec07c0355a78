// pi_ffn.cu -- C ABI of the predictor-gated sparse FFN decode library: host
// validation, workspace layout and kernel dispatch.  The declarations and
// argument contracts live in include/pi_ffn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "pi_batch.cuh"
#include "pi_ffn.h"
#include "pi_fused.cuh"
#include "pi_kernels.cuh"
#include "pi_tc.cuh"

struct pi_ffn {
  pi_ffn_desc d;
  int H;       // hot prefix rounded down to a multiple of 32
  int nwords;  // ceil(f / 32)
  // TMA tensor maps of the tensor-core path (valid when tc_maps)
  bool tc_maps;
  CUtensorMap tm_p1, tm_p2, tm_up, tm_gate, tm_down, ts_up, ts_gate, ts_down;
  // the batch-1 fused kernel's P2 tile map (valid when fx_ok, for fx_G CTAs)
  bool fx_ok;
  int fx_G, fx_M;
  CUtensorMap tm_p2_fused;
};

namespace {

constexpr int kMaxBatch = 32;
constexpr int kMaxD = 16384;

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace layout for a call at batch B on layers with the given maxima.
// [0, 256): status region: int status, int union count, grid-barrier word,
// at byte 64 the epoch of the fused kernel's tagged words, at byte 68 its
// arrival counter of the reduction slices.
// [256, 1024): the batch kernel's per-tile arrival counters (zero between
// calls; the kernel restores them), at a place that does not move with B.
// fx_h / fx_part: the fused kernel's tagged exchange words (h, partials of y);
// no other kernel writes them, so a stale word can never carry a current tag.
struct WsLayout {
  size_t h, u, mask, uwords, uprefix, ulist, partial, fx_h, fx_part, b_ahi, b_alo, b_part, total;
  int G, a_stride;
};
constexpr size_t kEpochOffset = 64;
constexpr size_t kTicketOffset = 68;
constexpr size_t kBatchCtrOffset = 256;
constexpr size_t kHeaderBytes = 1024;
static_assert(kBatchCtrOffset + pi::batch::kMaxTiles * 4 <= kHeaderBytes, "batch counters fit the header");

// A once-per-device setup step (a kernel's function attribute acts on the
// current device only): one bit per device ordinal below 64.
class DeviceOnce {
 public:
  // runs set() unless it already succeeded on the current device
  template <typename Set>
  cudaError_t ensure(Set set) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const unsigned long long bit = 1ull << dev;
    if (bits_.load(std::memory_order_acquire) & bit) return cudaSuccess;
    if ((e = set()) != cudaSuccess) return e;
    bits_.fetch_or(bit, std::memory_order_acq_rel);
    return cudaSuccess;
  }

 private:
  std::atomic<unsigned long long> bits_{0};
};

int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

WsLayout ws_layout(int dmax, int fmax, int rmax, int B, int G) {
  WsLayout L{};
  size_t o = kHeaderBytes;
  const size_t nw = (size_t)(fmax + 31) / 32;
  L.h = o;
  o = align_up(o + (size_t)B * rmax * 4, 256);
  L.u = o;
  o = align_up(o + (size_t)B * dmax * 2, 256);
  L.mask = o;
  o = align_up(o + (size_t)B * nw * 4, 256);
  L.uwords = o;
  o = align_up(o + nw * 4, 256);
  L.uprefix = o;
  o = align_up(o + (nw + 1) * 4, 256);
  L.ulist = o;
  o = align_up(o + (size_t)fmax * 4, 256);
  L.partial = o;
  o = align_up(o + (size_t)G * B * dmax * 4, 256);
  L.fx_h = o;
  o = align_up(o + (size_t)rmax * 8, 256);
  L.fx_part = o;
  o = align_up(o + (size_t)G * dmax * 8, 256);
  // batch kernel: activations by list position (hi and lo parts) and the
  // pieces of tiles split between CTAs
  // (batches of 2 or more only)
  L.a_stride = (int)align_up((size_t)fmax + pi::batch::kPosStep, 16);
  L.b_ahi = L.b_alo = L.b_part = o;
  if (B >= 2) {
    o = align_up(o + (size_t)pi::batch::kTok * L.a_stride * 2, 256);
    L.b_alo = o;
    o = align_up(o + (size_t)pi::batch::kTok * L.a_stride * 2, 256);
    L.b_part = o;
    o = align_up(o + (size_t)G * 2 * pi::batch::kPieceFloats * 4, 256);
  }
  L.total = o;
  L.G = G;
  return L;
}

// Tensor-core path (batch 16..32) scratch: token images, stream-K partials
// and per-tile counters.  It sits at the END of the caller's buffer so its
// counters keep their place whatever batch earlier calls used (they must stay
// zero between calls; the kernels restore them).
struct TcLayout {
  size_t uimg, uimg_perm, himg_hi, himg_lo, aimg, part, ctr_p1, ctr_p2, ctr_up, ctr_down, total;
};

TcLayout tc_layout(int dmax, int fmax, int rmax, int G) {
  TcLayout L{};
  size_t o = 0;
  const size_t step_img = (size_t)pi::tc::kImgStep / 16 * pi::tc::kBlk;
  L.uimg = o;
  o = align_up(o + (size_t)((dmax + 127) / 128) * step_img, 256);
  L.uimg_perm = o;
  o = align_up(o + (size_t)((dmax + 127) / 128) * step_img, 256);
  L.himg_hi = o;
  o = align_up(o + (size_t)((rmax + 127) / 128) * step_img, 256);
  L.himg_lo = o;
  o = align_up(o + (size_t)((rmax + 127) / 128) * step_img, 256);
  L.aimg = o;
  o = align_up(o + (size_t)((fmax + 127) / 128) * step_img, 256);
  L.part = o;
  o = align_up(o + (size_t)G * 2 * pi::tc::kPartFloats * 4, 256);
  L.ctr_p1 = o;
  o = align_up(o + (size_t)((rmax + 127) / 128) * 4, 256);
  L.ctr_p2 = o;
  o = align_up(o + (size_t)((fmax + 127) / 128) * 4, 256);
  L.ctr_up = o;
  o = align_up(o + (size_t)((fmax + 127) / 128) * 4, 256);
  L.ctr_down = o;
  o = align_up(o + (size_t)((dmax + pi::tc::kDownTileD - 1) / pi::tc::kDownTileD) * 4, 256);
  L.total = o;
  return L;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library); null when no driver is present.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encoder() {
  static EncodeTiledFn fn = []() -> EncodeTiledFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// 2D map of a row-major matrix [rows x inner] of 1- or 2-byte elements, box
// [box_rows x box_inner]; 128-byte swizzle when swz.  Outside reads are zero.
bool map_2d(CUtensorMap *m, const void *base, bool fp16, uint64_t inner, uint64_t rows, uint32_t box_inner,
            uint32_t box_rows, bool swz) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const uint64_t esz = fp16 ? 2 : 1;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * esz};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             swz ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor maps of the tcgen05 kernels: fp16 predictor; fp16 weights, or int4
// weights whose rows hold whole 256-element scale blocks.
bool build_tc_maps(pi_ffn *h) {
  const pi_ffn_desc &D = h->d;
  if (D.ptype != PI_W_F16) return false;
  const uint64_t d = D.d_model, f = D.d_ffn, r = D.rank;
  bool ok = map_2d(&h->tm_p1, D.p1, true, d, r, 64, 128, true) && map_2d(&h->tm_p2, D.p2, true, r, f, 64, 128, true);
  const bool swiglu = D.act == PI_ACT_SWIGLU;
  if (D.wtype == PI_W_F16) {
    ok = ok && map_2d(&h->tm_up, D.w_up, true, d, f, 64, 128, true) &&
         (!swiglu || map_2d(&h->tm_gate, D.w_gate, true, d, f, 64, 128, true)) &&
         map_2d(&h->tm_down, D.w_down_t, true, d, f, 64, 64, true);
  } else if (D.wtype == PI_W_INT4G32 && d % 256 == 0) {
    ok = ok && map_2d(&h->tm_up, D.w_up, false, d / 2, f, 128, 128, true) &&
         map_2d(&h->ts_up, D.s_up, false, d / 16, f, 16, 128, false) &&
         (!swiglu || (map_2d(&h->tm_gate, D.w_gate, false, d / 2, f, 128, 128, true) &&
                      map_2d(&h->ts_gate, D.s_gate, false, d / 16, f, 16, 128, false))) &&
         map_2d(&h->tm_down, D.w_down_t, false, d / 2, f, 128, 64, true) &&
         map_2d(&h->ts_down, D.s_down_t, false, d / 16, f, 16, 64, false);
  } else {
    ok = false;
  }
  return ok;
}

// The fused kernel's view of P2: the 4D tensor (k % 8, m, k / 8, c) of the
// element k of neuron c + m G, for the G CTAs of one SM each and m < f / G,
// so that one box {8, 32, r / 8, 1} brings a CTA's 32-row tile in the
// K-interleaved order its ldmatrix reads.  Elements with m >= f / G read as
// zero; the remaining f mod G rows are copied one per CTA.
bool build_fused_map(pi_ffn *h) {
  const pi_ffn_desc &D = h->d;
  h->fx_ok = false;
  const int G = device_sm_count();
  if (G <= 0 || D.ptype != PI_W_F16 || D.rank % 16 || D.rank > 1024) return false;
  h->fx_G = G;
  h->fx_M = D.d_ffn / G;
  if (h->fx_M == 0) return h->fx_ok = true;  // every row is a leftover row: no map
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const uint64_t r = (uint64_t)D.rank;
  const cuuint64_t dims[4] = {8, (cuuint64_t)h->fx_M, r / 8, (cuuint64_t)G};
  const cuuint64_t strides[3] = {(cuuint64_t)G * r * 2, 16, r * 2};
  const cuuint32_t box[4] = {8, 32, (cuuint32_t)(r / 8), 1};
  const cuuint32_t es[4] = {1, 1, 1, 1};
  h->fx_ok = enc(&h->tm_p2_fused, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void *>(D.p2), dims, strides, box,
                 es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  return h->fx_ok;
}

// Smallest batch that takes the tensor-core path: int4 layers from 2 tokens
// (the CUDA-core batch kernel reads fp16 rows only), fp16 layers from 9 (the
// CUDA-core batch kernel covers 2..8).
int tc_min_batch(const pi_ffn *h) { return h->d.wtype == PI_W_INT4G32 ? 2 : 9; }
bool tc_ok(const pi_ffn *h, int B);

struct Ws {
  WsLayout L;
  TcLayout T;
  char *base;
  char *tc;  // start of the tensor-core region (null when the call does not use it)
  int *status() const { return reinterpret_cast<int *>(base); }
  int32_t *ucount() const { return reinterpret_cast<int32_t *>(base) + 1; }
  unsigned *grid_bar() const { return reinterpret_cast<unsigned *>(base) + 2; }
  float *h() const { return reinterpret_cast<float *>(base + L.h); }
  __half *u() const { return reinterpret_cast<__half *>(base + L.u); }
  uint32_t *mask() const { return reinterpret_cast<uint32_t *>(base + L.mask); }
  uint32_t *uwords() const { return reinterpret_cast<uint32_t *>(base + L.uwords); }
  int32_t *uprefix() const { return reinterpret_cast<int32_t *>(base + L.uprefix); }
  int32_t *ulist() const { return reinterpret_cast<int32_t *>(base + L.ulist); }
  float *partial() const { return reinterpret_cast<float *>(base + L.partial); }
  unsigned *epoch() const { return reinterpret_cast<unsigned *>(base + kEpochOffset); }
  unsigned *ticket() const { return reinterpret_cast<unsigned *>(base + kTicketOffset); }
  unsigned long long *fx_h() const { return reinterpret_cast<unsigned long long *>(base + L.fx_h); }
  unsigned long long *fx_part() const { return reinterpret_cast<unsigned long long *>(base + L.fx_part); }
  __half *b_ahi() const { return reinterpret_cast<__half *>(base + L.b_ahi); }
  __half *b_alo() const { return reinterpret_cast<__half *>(base + L.b_alo); }
  float *b_part() const { return reinterpret_cast<float *>(base + L.b_part); }
  unsigned *b_ctr() const { return reinterpret_cast<unsigned *>(base + kBatchCtrOffset); }
  unsigned char *uimg() const { return reinterpret_cast<unsigned char *>(tc + T.uimg); }
  unsigned char *uimg_perm() const { return reinterpret_cast<unsigned char *>(tc + T.uimg_perm); }
  unsigned char *himg_hi() const { return reinterpret_cast<unsigned char *>(tc + T.himg_hi); }
  unsigned char *himg_lo() const { return reinterpret_cast<unsigned char *>(tc + T.himg_lo); }
  unsigned char *aimg() const { return reinterpret_cast<unsigned char *>(tc + T.aimg); }
  float *tc_part() const { return reinterpret_cast<float *>(tc + T.part); }
  int *ctr_p1() const { return reinterpret_cast<int *>(tc + T.ctr_p1); }
  int *ctr_p2() const { return reinterpret_cast<int *>(tc + T.ctr_p2); }
  int *ctr_up() const { return reinterpret_cast<int *>(tc + T.ctr_up); }
  int *ctr_down() const { return reinterpret_cast<int *>(tc + T.ctr_down); }
};

pi_status get_ws(const pi_ffn *const *layers, int n, int B, void *ws, size_t ws_bytes, Ws *out) {
  if (!ws) return PI_ERR_WORKSPACE;
  if (!aligned16(ws)) return PI_ERR_MISALIGNED;
  int dmax = 0, fmax = 0, rmax = 0;
  for (int i = 0; i < n; ++i) {
    dmax = dmax > layers[i]->d.d_model ? dmax : layers[i]->d.d_model;
    fmax = fmax > layers[i]->d.d_ffn ? fmax : layers[i]->d.d_ffn;
    rmax = rmax > layers[i]->d.rank ? rmax : layers[i]->d.rank;
  }
  const int G = device_sm_count();
  if (G <= 0) return PI_ERR_CUDA;
  out->L = ws_layout(dmax, fmax, rmax, B, G);
  out->base = static_cast<char *>(ws);
  out->tc = nullptr;
  bool tc = false;
  for (int i = 0; i < n; ++i) tc = tc || tc_ok(layers[i], B);
  if (tc) {
    out->T = tc_layout(dmax, fmax, rmax, G);
    if (out->T.total > ws_bytes) return PI_ERR_WORKSPACE;
    const uintptr_t end = reinterpret_cast<uintptr_t>(ws) + ws_bytes;
    const uintptr_t tc = (end - out->T.total) & ~(uintptr_t)255;
    if (tc < reinterpret_cast<uintptr_t>(ws) + out->L.total) return PI_ERR_WORKSPACE;
    out->tc = reinterpret_cast<char *>(tc);
    return PI_OK;
  }
  return out->L.total <= ws_bytes ? PI_OK : PI_ERR_WORKSPACE;
}

// ---------------------------------------------------------------- launching
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*kern)(KArgs...), dim3 grid, dim3 block, cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

inline int nb_for(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 8; }
inline int cdiv(int a, int b) { return (a + b - 1) / b; }

template <int NB>
cudaError_t pred_h_nb(int pt, dim3 g, cudaStream_t st, const void *p1, const void *u, int d, int r, int B, float *h) {
  return pt == PI_W_F32 ? launch(pi::pred_h_kernel<NB, pi::W_F32>, g, dim3(256), st, p1, u, d, r, B, h)
                        : launch(pi::pred_h_kernel<NB, pi::W_F16>, g, dim3(256), st, p1, u, d, r, B, h);
}
template <int NB>
cudaError_t pred_s_nb(int pt, dim3 g, cudaStream_t st, const void *p2, const float *h, const float *bias, int f, int r,
                      int B, uint32_t *mask, int nw) {
  return pt == PI_W_F32 ? launch(pi::pred_s_kernel<NB, pi::W_F32>, g, dim3(256), st, p2, h, bias, f, r, B, mask, nw)
                        : launch(pi::pred_s_kernel<NB, pi::W_F16>, g, dim3(256), st, p2, h, bias, f, r, B, mask, nw);
}

// gather kernel dispatch: NB tokens per CTA row, GPT column groups per thread
template <int NB, int WT, int ACT>
cudaError_t gather_gpt(int gpt, dim3 g, dim3 b, cudaStream_t st, const pi::FfnArgs &a) {
  switch (gpt) {
  case 1:
    return launch(pi::ffn_gather_kernel<NB, WT, ACT, 1>, g, b, st, a);
  case 2:
    if constexpr (NB * 2 <= 8) return launch(pi::ffn_gather_kernel<NB, WT, ACT, 2>, g, b, st, a);
    break;
  case 4:
    if constexpr (NB * 4 <= 8) return launch(pi::ffn_gather_kernel<NB, WT, ACT, 4>, g, b, st, a);
    break;
  }
  return cudaErrorInvalidConfiguration;
}
template <int NB, int WT>
cudaError_t gather_act(int act, int gpt, dim3 g, dim3 b, cudaStream_t st, const pi::FfnArgs &a) {
  return act == PI_ACT_RELU ? gather_gpt<NB, WT, pi::ACT_RELU>(gpt, g, b, st, a)
                            : gather_gpt<NB, WT, pi::ACT_SWIGLU>(gpt, g, b, st, a);
}
template <int NB>
cudaError_t gather_wt(int wt, int act, int gpt, dim3 g, dim3 b, cudaStream_t st, const pi::FfnArgs &a) {
  switch (wt) {
  case PI_W_F32:
    return gather_act<NB, pi::W_F32>(act, gpt, g, b, st, a);
  case PI_W_F16:
    return gather_act<NB, pi::W_F16>(act, gpt, g, b, st, a);
  default:
    return gather_act<NB, pi::W_INT4>(act, gpt, g, b, st, a);
  }
}

// Token group size and column groups per thread for the gather kernel:
// NB * GPT <= 8 (at most 64 fp32 accumulators per thread) and the CTA covers
// the d/8 column groups with at most 512 threads (128 registers each).
void gather_shape(int B, int d, int *nb, int *gpt, int *threads) {
  const int ngroups = d / 8;
  for (int n = nb_for(B); n >= 1; n >>= 1) {
    for (int g = 1; g <= 4 && n * g <= 8; g <<= 1) {
      const int maxt = 512;
      int t = (cdiv(ngroups, g) + 31) / 32 * 32;
      if (t < 128) t = 128;
      if (t <= maxt) {
        *nb = n;
        *gpt = g;
        *threads = t;
        return;
      }
    }
  }
  *nb = 1;
  *gpt = 4;
  *threads = 512;
}

bool want_dense(const pi_ffn *h, int B, unsigned flags) {
  if (h->H <= 0) return false;
  if (flags & PI_FFN_HOT_DENSE) return true;
  if (flags & PI_FFN_HOT_INDEX) return false;
  const double p = h->d.hot_p_mean;
  if (!(p > 0.0)) return false;
  return 1.0 - std::pow(1.0 - (p < 1.0 ? p : 1.0), (double)B) >= 0.75;
}

#define PI_CUDA(call)                      \
  do {                                     \
    if ((call) != cudaSuccess) return PI_ERR_CUDA; \
  } while (0)

// Test support (pi_debug_wait_fault): an entry of h that is never published,
// and a shorter limit for every bounded wait of the fused and batch
// kernels.
struct WaitFault {
  int withhold = -1;
  unsigned long long limit_ns = 0;  // 0: the kernel's default
};
WaitFault g_wait_fault;

// The tensor-core predictor kernels of batches 2..8: fp16 predictor, rank a
// multiple of 64 up to 1024, d a multiple of 64 up to 8192, P1 and P2 on
// 32-byte boundaries (256-bit row loads).
bool pred_batch_ok(const pi_ffn *h, int B) {
  const pi_ffn_desc &D = h->d;
  if (B < 2 || B > pi::batch::kTok || D.ptype != PI_W_F16) return false;
  if (D.rank % 64 || D.rank > 64 * 8 * pi::batch::kPredSUnits) return false;
  if (D.d_model % 64 || D.d_model > 64 * pi::batch::kWarps * pi::batch::kPredHUnits) return false;
  // one CTA per SM computes 8 rows of h
  if (D.rank > pi::batch::kPredHRows * device_sm_count()) return false;
  return !((reinterpret_cast<uintptr_t>(D.p1) | reinterpret_cast<uintptr_t>(D.p2)) & 31u);
}

bool batch_ok(const pi_ffn *h, int B, int G);
bool tc_ok(const pi_ffn *h, int B);

// steps 1-2: predictor, mask words, compaction (idx/count optional; the batch
// FFN kernel scans the union words itself, so without lists it needs none)
pi_status run_predict(const pi_ffn *h, const void *u, int B, int32_t *idx, int idx_stride, int32_t *count, const Ws &w,
                      cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  if (pred_batch_ok(h, B)) {
    pi::batch::PredArgs a{};
    a.p1 = reinterpret_cast<const __half *>(D.p1);
    a.p2 = reinterpret_cast<const __half *>(D.p2);
    a.p_bias = D.p_bias;
    a.u = reinterpret_cast<const __half *>(u);
    a.h = w.h();
    a.d = D.d_model;
    a.r = D.rank;
    a.f = D.d_ffn;
    a.B = B;
    a.mask = w.mask();
    a.uwords = w.uwords();
    a.nwords = h->nwords;
    a.bar = w.grid_bar();
    a.status = w.status();
    a.wait_ns = g_wait_fault.limit_ns ? g_wait_fault.limit_ns : pi::batch::kWaitNs;
    PI_CUDA(launch(pi::batch::pred_batch_kernel, dim3(w.L.G), dim3(pi::batch::kThreads), st, a));
    // the batch FFN kernel scans the union words itself and the tensor-core
    // FFN kernels list their tiles from them: only the multi-kernel gather
    // needs the compacted list
    if (idx || count || !(batch_ok(h, B, w.L.G) || tc_ok(h, B)))
      PI_CUDA(launch(pi::compact_kernel, dim3(B + 1), dim3(1024), st, (const uint32_t *)w.mask(), h->nwords,
                     idx_stride, B, idx, count, w.uwords(), w.uprefix(), w.ulist(), w.ucount()));
    return PI_OK;
  }
  const int nb = nb_for(B);
  const dim3 gh(cdiv(D.rank, 8), cdiv(B, nb)), gs(h->nwords, cdiv(B, nb));
  cudaError_t e;
  switch (nb) {
  case 1:
    e = pred_h_nb<1>(D.ptype, gh, st, D.p1, u, D.d_model, D.rank, B, w.h());
    break;
  case 2:
    e = pred_h_nb<2>(D.ptype, gh, st, D.p1, u, D.d_model, D.rank, B, w.h());
    break;
  case 4:
    e = pred_h_nb<4>(D.ptype, gh, st, D.p1, u, D.d_model, D.rank, B, w.h());
    break;
  default:
    e = pred_h_nb<8>(D.ptype, gh, st, D.p1, u, D.d_model, D.rank, B, w.h());
  }
  PI_CUDA(e);
  switch (nb) {
  case 1:
    e = pred_s_nb<1>(D.ptype, gs, st, D.p2, w.h(), D.p_bias, D.d_ffn, D.rank, B, w.mask(), h->nwords);
    break;
  case 2:
    e = pred_s_nb<2>(D.ptype, gs, st, D.p2, w.h(), D.p_bias, D.d_ffn, D.rank, B, w.mask(), h->nwords);
    break;
  case 4:
    e = pred_s_nb<4>(D.ptype, gs, st, D.p2, w.h(), D.p_bias, D.d_ffn, D.rank, B, w.mask(), h->nwords);
    break;
  default:
    e = pred_s_nb<8>(D.ptype, gs, st, D.p2, w.h(), D.p_bias, D.d_ffn, D.rank, B, w.mask(), h->nwords);
  }
  PI_CUDA(e);
  PI_CUDA(launch(pi::compact_kernel, dim3(B + 1), dim3(1024), st, (const uint32_t *)w.mask(), h->nwords, idx_stride, B,
                 idx, count, w.uwords(), w.uprefix(), w.ulist(), w.ucount()));
  return PI_OK;
}

// caller id lists -> mask words and union
pi_status run_sets(const pi_ffn *h, const int32_t *idx, const int32_t *count, int B, const Ws &w, cudaStream_t st) {
  PI_CUDA(cudaMemsetAsync(w.mask(), 0, (size_t)B * h->nwords * 4, st));
  const int f = h->d.d_ffn;
  PI_CUDA(launch(pi::idx_to_mask_kernel, dim3(cdiv(f, 256) < 64 ? cdiv(f, 256) : 64, B), dim3(256), st, idx, count, f,
                 w.mask(), h->nwords, w.status()));
  PI_CUDA(launch(pi::compact_kernel, dim3(B + 1), dim3(1024), st, (const uint32_t *)w.mask(), h->nwords, 0, B,
                 (int32_t *)nullptr, (int32_t *)nullptr, w.uwords(), w.uprefix(), w.ulist(), w.ucount()));
  return PI_OK;
}


// ---------------------------------------------------------------- batch kernel (2..8 tokens)
namespace BK = pi::batch;

// The batch kernel takes fp16 weights with d a multiple of 64 (d <= 12288),
// up / gate matrices on 32-byte boundaries (256-bit row loads), 2..8 tokens,
// and at most kMaxLoc list positions per CTA.
bool batch_ok(const pi_ffn *h, int B, int G) {
  const pi_ffn_desc &D = h->d;
  if (B < 2 || B > BK::kTok || D.wtype != PI_W_F16) return false;
  if ((reinterpret_cast<uintptr_t>(D.w_up) & 31u) || (D.w_gate && (reinterpret_cast<uintptr_t>(D.w_gate) & 31u)))
    return false;
  if (D.d_model % BK::kTileCols || D.d_model / BK::kTileCols > BK::kMaxTiles) return false;
  if (h->nwords > BK::kMaxWords) return false;
  const int nm = D.act == PI_ACT_SWIGLU ? 2 : 1;
  if (BK::smem_bytes(D.d_model, nm) > 200 * 1024) return false;
  return (D.d_ffn + G - 1) / G <= BK::kMaxLoc;
}

template <int ACT>
cudaError_t batch_launch(const BK::Args &a, int G, int d, cudaStream_t st) {
  static DeviceOnce attr;
  const int smem = (int)BK::smem_bytes(d, ACT == pi::ACT_SWIGLU ? 2 : 1);
  // the largest size any layer may take (batch_ok), set once per device
  cudaError_t e = attr.ensure([] {
    return cudaFuncSetAttribute(BK::ffn_batch_kernel<ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(BK::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // programmatic dependent launch, no cooperative attribute: one CTA per SM,
  // and the one grid-wide wait is bounded (PI_ERR_TIMEOUT, never a hang)
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, BK::ffn_batch_kernel<ACT>, a);
}

pi_status run_ffn_batch(const pi_ffn *h, const void *u, int B, float *out, int accumulate, unsigned flags,
                        const Ws &w, cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  BK::Args a{};
  a.w_up = D.w_up;
  a.w_gate = D.w_gate;
  a.w_down_t = D.w_down_t;
  a.b_up = D.b_up;
  a.u = reinterpret_cast<const __half *>(u);
  a.d = D.d_model;
  a.f = D.d_ffn;
  a.B = B;
  a.mask = w.mask();
  a.uwords = w.uwords();
  a.nwords = h->nwords;
  a.ulist = w.ulist();
  a.hot_dense = want_dense(h, B, flags) ? 1 : 0;
  a.H = h->H;
  a.a_hi = w.b_ahi();
  a.a_lo = w.b_alo();
  a.a_stride = w.L.a_stride;
  a.part = w.b_part();
  a.ctr = w.b_ctr();
  a.bar = w.grid_bar();
  a.out = out;
  a.accumulate = accumulate;
  a.status = w.status();
  a.wait_ns = g_wait_fault.limit_ns ? g_wait_fault.limit_ns : BK::kWaitNs;
  const cudaError_t e = D.act == PI_ACT_RELU ? batch_launch<pi::ACT_RELU>(a, w.L.G, D.d_model, st)
                                             : batch_launch<pi::ACT_SWIGLU>(a, w.L.G, D.d_model, st);
  return e == cudaSuccess ? PI_OK : PI_ERR_CUDA;
}

// steps 3-4 over the union in the workspace; out (=, +=) y
pi_status run_ffn(const pi_ffn *h, const void *u, int B, float *out, int accumulate, unsigned flags, const Ws &w,
                  cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  if (batch_ok(h, B, w.L.G)) return run_ffn_batch(h, u, B, out, accumulate, flags, w, st);
  pi::FfnArgs a{};
  a.w_up = D.w_up;
  a.w_gate = D.w_gate;
  a.w_down_t = D.w_down_t;
  a.s_up = reinterpret_cast<const __half *>(D.s_up);
  a.s_gate = reinterpret_cast<const __half *>(D.s_gate);
  a.s_down_t = reinterpret_cast<const __half *>(D.s_down_t);
  a.b_up = D.b_up;
  a.u = u;
  a.d = D.d_model;
  a.f = D.d_ffn;
  a.B = B;
  a.mask = w.mask();
  a.nwords = h->nwords;
  a.ulist = w.ulist();
  a.ucount = w.ucount();
  a.uprefix = w.uprefix();
  a.hot_dense = want_dense(h, B, flags) ? 1 : 0;
  a.H = h->H;
  a.partial = w.partial();
  int nb, gpt, threads;
  gather_shape(B, D.d_model, &nb, &gpt, &threads);
  const dim3 g(w.L.G, cdiv(B, nb)), blk(threads);
  cudaError_t e;
  switch (nb) {
  case 1:
    e = gather_wt<1>(D.wtype, D.act, gpt, g, blk, st, a);
    break;
  case 2:
    e = gather_wt<2>(D.wtype, D.act, gpt, g, blk, st, a);
    break;
  case 4:
    e = gather_wt<4>(D.wtype, D.act, gpt, g, blk, st, a);
    break;
  default:
    e = gather_wt<8>(D.wtype, D.act, gpt, g, blk, st, a);
  }
  PI_CUDA(e);
  const int n_elem = B * D.d_model;
  PI_CUDA(launch(pi::reduce_kernel, dim3(cdiv(n_elem, 32)), dim3(256), st, (const float *)w.partial(), w.L.G, n_elem,
                 out, accumulate));
  return PI_OK;
}

// ---------------------------------------------------------------- tensor-core path (batch 16..32)
namespace TC = pi::tc;

// The tcgen05 kernels take fp16 predictors and fp16 or int4 weights (int4
// rows in whole 256-element scale blocks; see build_tc_maps) at
// tc_min_batch <= B <= 32 (token columns past B are zero).
bool tc_ok(const pi_ffn *h, int B) {
  return B >= tc_min_batch(h) && B <= TC::kN && h->tc_maps && h->d.d_ffn <= TC::kMaxTiles * TC::kM;
}

template <typename KArg>
cudaError_t launch_smem(void (*kern)(KArg), int G, int threads, int smem, DeviceOnce *attr, cudaStream_t st,
                        const KArg &arg) {
  cudaError_t e =
      attr->ensure([&] { return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, arg);
}

template <int KIND, int WT, int ACT>
cudaError_t ts_launch(const TC::RowArgs &a, int G, cudaStream_t st) {
  static DeviceOnce attr;
  using Sh = TC::RowShape<KIND, WT, ACT>;
  return launch_smem(TC::row_gemm_kernel<KIND, WT, ACT>, G, Sh::THREADS, Sh::SMEM, &attr, st, a);
}

template <int WT>
cudaError_t down_launch(const TC::DownArgs &a, int G, cudaStream_t st) {
  static DeviceOnce attr;
  return launch_smem(TC::ffn_down_kernel<WT>, G, TC::kThreads, TC::DownShape<WT>::SMEM, &attr, st, a);
}

// token images of u: natural order (predictor, fp16 weights) and, for int4
// weights, the paired order of the int4 up/gate dequantisation
cudaError_t tc_u_image(const pi_ffn *h, const void *u, int B, const Ws &w, cudaStream_t st) {
  const int d = h->d.d_model;
  const int total = TC::kN * ((d + 127) / 128) * 16;
  unsigned char *perm = h->d.wtype == PI_W_INT4G32 ? w.uimg_perm() : nullptr;
  return launch(TC::u_image_kernel, dim3(cdiv(total, 256)), dim3(256), st, (const __half *)u, B, d, w.uimg(), perm);
}

// steps 1-2 on tensor cores: u image, h = P1 u (hi/lo images), mask words, compaction
pi_status run_predict_tc(const pi_ffn *h, const void *u, int B, int32_t *idx, int idx_stride, int32_t *count,
                         const Ws &w, cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  const int G = w.L.G;
  PI_CUDA(tc_u_image(h, u, B, w, st));
  TC::RowArgs a{};
  a.tm0 = h->tm_p1;
  a.nrows = D.rank;
  a.K = D.d_model;
  a.img0 = w.uimg();
  a.out0 = w.himg_hi();
  a.out1 = w.himg_lo();
  a.uwords = w.uwords();
  a.nwords = h->nwords;
  a.B = B;
  a.part = w.tc_part();
  a.ctr = w.ctr_p1();
  a.status = w.status();
  PI_CUDA((ts_launch<TC::K_P1, pi::W_F16, 0>(a, G, st)));
  TC::RowArgs b{};
  b.tm0 = h->tm_p2;
  b.nrows = D.d_ffn;
  b.K = D.rank;
  b.img0 = w.himg_hi();
  b.img1 = w.himg_lo();
  b.bias = D.p_bias;
  b.mask_out = w.mask();
  b.uwords = w.uwords();
  b.nwords = h->nwords;
  b.B = B;
  b.part = w.tc_part();
  b.ctr = w.ctr_p2();
  b.status = w.status();
  PI_CUDA((ts_launch<TC::K_P2, pi::W_F16, 0>(b, G, st)));
  // pred_h clears and pred_s sets the union words the tensor-core FFN kernels
  // list their tiles from; the compaction runs only for the caller's id lists
  if (idx || count)
    PI_CUDA(launch(pi::compact_kernel, dim3(B + 1), dim3(1024), st, (const uint32_t *)w.mask(), h->nwords, idx_stride,
                   B, idx, count, w.uwords(), w.uprefix(), w.ulist(), w.ucount()));
  return PI_OK;
}

// steps 3-4 on tensor cores over the union in the workspace; out (=, +=) y
pi_status run_ffn_tc(const pi_ffn *h, const void *u, int B, float *out, int accumulate, bool u_ready, const Ws &w,
                     cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  const int G = w.L.G;
  if (!u_ready) PI_CUDA(tc_u_image(h, u, B, w, st));
  TC::RowArgs a{};
  a.tm0 = h->tm_up;
  a.tm1 = h->tm_gate;
  a.ts0 = h->ts_up;
  a.ts1 = h->ts_gate;
  a.uwords = w.uwords();
  a.nrows = D.d_ffn;
  a.K = D.d_model;
  a.img0 = D.wtype == PI_W_INT4G32 ? w.uimg_perm() : w.uimg();
  a.bias = D.b_up;
  a.mask = w.mask();
  a.nwords = h->nwords;
  a.B = B;
  a.out0 = w.aimg();
  a.part = w.tc_part();
  a.ctr = w.ctr_up();
  a.status = w.status();
  const bool relu = D.act == PI_ACT_RELU;
  cudaError_t e;
  if (D.wtype == PI_W_F16)
    e = relu ? ts_launch<TC::K_UP, pi::W_F16, pi::ACT_RELU>(a, G, st)
             : ts_launch<TC::K_UP, pi::W_F16, pi::ACT_SWIGLU>(a, G, st);
  else
    e = relu ? ts_launch<TC::K_UP, pi::W_INT4, pi::ACT_RELU>(a, G, st)
             : ts_launch<TC::K_UP, pi::W_INT4, pi::ACT_SWIGLU>(a, G, st);
  PI_CUDA(e);
  TC::DownArgs dn{};
  dn.tm = h->tm_down;
  dn.ts = h->ts_down;
  dn.uwords = w.uwords();
  dn.nwords = h->nwords;
  dn.f = D.d_ffn;
  dn.d = D.d_model;
  dn.B = B;
  dn.aimg = w.aimg();
  dn.y = out;
  dn.accumulate = accumulate;
  dn.part = w.tc_part();
  dn.ctr = w.ctr_down();
  dn.status = w.status();
  PI_CUDA(D.wtype == PI_W_F16 ? down_launch<pi::W_F16>(dn, G, st) : down_launch<pi::W_INT4>(dn, G, st));
  return PI_OK;
}

// ---------------------------------------------------------------- fused batch-1 path
namespace F = pi::fused;


template <int WT, int ACT, int CPT>
cudaError_t fused_launch(const F::Args &a, int G, cudaStream_t st) {
  static DeviceOnce attr;
  const size_t smem = sizeof(F::Smem);
  cudaError_t e = attr.ensure([&] {
    cudaError_t r = cudaFuncSetAttribute(F::decode_fused_kernel<WT, ACT, CPT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (r != cudaSuccess) return r;
    int nb = 0;
    r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, F::decode_fused_kernel<WT, ACT, CPT>, F::kThreads, smem);
    if (r != cudaSuccess) return r;
    return nb < 1 ? cudaErrorInvalidConfiguration : cudaSuccess;
  });
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(G);
  cfg.blockDim = dim3(F::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  // Programmatic dependent launch, and no cooperative attribute: a
  // cooperative grid is only scheduled once every SM is free, while here the
  // CTAs of the next launch take the SMs of this launch's CTAs as they leave
  // and start streaming weights during its reduction.  The grid is one CTA per
  // SM and every wait for another CTA is bounded, so CTAs that cannot all be
  // resident (another kernel holding SMs for longer than the limit) end in
  // PI_ERR_TIMEOUT, never in a hang.
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, F::decode_fused_kernel<WT, ACT, CPT>, a);
}

// The fused kernel covers batch 1 with fp16 or int4 weights, d <= 8192, an
// fp16 predictor of rank <= 1024, and one neuron's rows fitting one slot.
bool fused_ok(const pi_ffn *h, int B, int G) {
  const pi_ffn_desc &D = h->d;
  if (B != 1 || D.ptype != PI_W_F16 || D.rank > F::kMaxR || D.rank % 16 || G > 320) return false;
  if (!h->fx_ok || h->fx_G != G) return false;
  if (D.wtype == PI_W_F16) {
    if (D.d_model > 8192) return false;
  } else if (D.wtype == PI_W_INT4G32) {
    if (D.d_model > 8192 || D.d_model % 256) return false;
  } else {
    return false;
  }
  const long rb = D.wtype == PI_W_F16 ? 2L * D.d_model : D.d_model / 2;
  const long sb = D.wtype == PI_W_INT4G32 ? D.d_model / 16 : 0;
  const int nmat = D.act == PI_ACT_SWIGLU ? 3 : 2;
  if (nmat * (rb + sb) > F::kSlotBytes) return false;
  const int per_cta = (D.d_ffn + G - 1) / G;  // neurons dealt to one CTA
  return (per_cta + F::kTN - 1) / F::kTN <= F::kMaxOwnTiles;
}

pi_status run_fused(const pi_ffn *h, const void *in, float *out, int stack, int accumulate, int32_t *idx,
                    int32_t *count, unsigned flags, const Ws &w, cudaStream_t st) {
  const pi_ffn_desc &D = h->d;
  F::Args a{};
  a.tm_p2 = h->tm_p2_fused;
  a.p2_main = h->fx_M;
  a.w_up = D.w_up;
  a.w_gate = D.w_gate;
  a.w_down_t = D.w_down_t;
  a.s_up = reinterpret_cast<const __half *>(D.s_up);
  a.s_gate = reinterpret_cast<const __half *>(D.s_gate);
  a.s_down_t = reinterpret_cast<const __half *>(D.s_down_t);
  a.b_up = D.b_up;
  a.p1 = reinterpret_cast<const __half *>(D.p1);
  a.p2 = reinterpret_cast<const __half *>(D.p2);
  a.p_bias = D.p_bias;
  a.in = in;
  a.out = out;
  a.d = D.d_model;
  a.f = D.d_ffn;
  a.r = D.rank;
  a.stack = stack;
  a.accumulate = accumulate;
  a.H = want_dense(h, 1, flags) ? h->H : 0;
  a.hx = w.fx_h();
  a.px = w.fx_part();
  a.epoch = w.epoch();
  a.ticket = w.ticket();
  a.mask32 = w.mask();
  a.bar = w.grid_bar();
  a.status = w.status();
  a.idx = idx;
  a.count = count;
  a.wait_ns = g_wait_fault.limit_ns ? g_wait_fault.limit_ns : F::kWaitNs;
  a.withhold = g_wait_fault.withhold;
  cudaError_t e;
  const bool relu = D.act == PI_ACT_RELU;
  const int G = w.L.G;
  if (D.wtype == PI_W_F16) {
    if (D.d_model <= F::kConsumers * 8)
      e = relu ? fused_launch<pi::W_F16, pi::ACT_RELU, 1>(a, G, st) : fused_launch<pi::W_F16, pi::ACT_SWIGLU, 1>(a, G, st);
    else
      e = relu ? fused_launch<pi::W_F16, pi::ACT_RELU, 2>(a, G, st) : fused_launch<pi::W_F16, pi::ACT_SWIGLU, 2>(a, G, st);
  } else {
    e = relu ? fused_launch<pi::W_INT4, pi::ACT_RELU, 1>(a, G, st)
             : fused_launch<pi::W_INT4, pi::ACT_SWIGLU, 1>(a, G, st);
  }
  return e == cudaSuccess ? PI_OK : PI_ERR_CUDA;
}

pi_status check_call(const pi_ffn *h, int B) {
  if (!h) return PI_ERR_INVALID_ARG;
  if (B < 0 || B > kMaxBatch) return PI_ERR_UNSUPPORTED;
  return PI_OK;
}

}  // namespace

// ---------------------------------------------------------------- static scratch
// Device scratch for pi_decode_ffn_static, for callers that cannot allocate
// device memory at decode time (no allocator handle of their own, HBM fully
// reserved by their caching allocator, or no tolerance for cudaMalloc's
// implicit device synchronisation).  One array per device, loaded with the
// module; it is laid out like a batch-1 workspace.
static __device__ __align__(256) unsigned char g_static_scratch[PI_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxStaticDevices = 64;
std::mutex g_static_mu;
struct StaticEntry {
  void *ctx = nullptr;  // context the address belongs to
  void *ptr = nullptr;
};
StaticEntry g_static[kMaxStaticDevices];

// The current context (cuCtxGetCurrent through the runtime's driver entry
// point), so that a cached address is reused only inside the context it was
// looked up in: a device reset or a new primary context reloads the module,
// and the array can move.
using CtxGetCurrentFn = CUresult (*)(CUcontext *);
void *current_context() {
  static CtxGetCurrentFn fn = []() -> CtxGetCurrentFn {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p) {
      cudaGetLastError();
      return nullptr;
    }
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device address of the scratch array on the current device, looked up with
// that device current the first time a context uses it, then cached for the
// context.
pi_status static_scratch(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return PI_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticDevices) return PI_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  void *ctx = current_context();
  StaticEntry &e = g_static[dev];
  if (!e.ptr || !ctx || e.ctx != ctx) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return PI_ERR_CUDA;
    e.ptr = p;
    e.ctx = current_context();  // the lookup makes the primary context current if none was
  }
  *out = e.ptr;
  return PI_OK;
}

}  // namespace

// ====================================================================== API

extern "C" {

pi_status pi_ffn_create(const pi_ffn_desc *desc, pi_ffn_t *out) {
  if (!desc || !out) return PI_ERR_INVALID_ARG;
  const pi_ffn_desc &D = *desc;
  if (D.d_model <= 0 || D.d_ffn <= 0 || D.rank <= 0) return PI_ERR_INVALID_ARG;
  if (D.act != PI_ACT_RELU && D.act != PI_ACT_SWIGLU) return PI_ERR_INVALID_ARG;
  if (D.wtype != PI_W_F32 && D.wtype != PI_W_F16 && D.wtype != PI_W_INT4G32) return PI_ERR_INVALID_ARG;
  if (D.ptype != PI_W_F32 && D.ptype != PI_W_F16) return PI_ERR_INVALID_ARG;
  if (!D.w_up || !D.w_down_t || !D.p1 || !D.p2 || !D.p_bias) return PI_ERR_INVALID_ARG;
  if (D.act == PI_ACT_RELU && !D.b_up) return PI_ERR_INVALID_ARG;
  if (D.act == PI_ACT_SWIGLU && !D.w_gate) return PI_ERR_INVALID_ARG;
  if (D.wtype == PI_W_INT4G32 && (!D.s_up || !D.s_down_t || (D.act == PI_ACT_SWIGLU && !D.s_gate)))
    return PI_ERR_INVALID_ARG;
  if (D.hot_prefix < 0 || D.hot_prefix > D.d_ffn) return PI_ERR_INVALID_ARG;
  // the FFN input u is fp32 exactly when the weights are fp32; the predictor
  // factors share u's type
  if ((D.wtype == PI_W_F32) != (D.ptype == PI_W_F32)) return PI_ERR_UNSUPPORTED;
  if (D.d_model % 8 || D.d_model > kMaxD) return PI_ERR_UNSUPPORTED;
  if (D.wtype == PI_W_INT4G32 && D.d_model % 32) return PI_ERR_UNSUPPORTED;
  if (D.rank % (D.ptype == PI_W_F32 ? 4 : 8)) return PI_ERR_UNSUPPORTED;
  const void *ptrs[] = {D.w_up, D.w_gate, D.w_down_t, D.s_up, D.s_gate, D.s_down_t, D.b_up, D.p1, D.p2, D.p_bias};
  for (const void *p : ptrs)
    if (p && !aligned16(p)) return PI_ERR_MISALIGNED;
  pi_ffn *h = new (std::nothrow) pi_ffn;
  if (!h) return PI_ERR_INVALID_ARG;
  h->d = D;
  h->H = D.hot_prefix & ~31;
  h->nwords = (D.d_ffn + 31) / 32;
  h->tc_maps = build_tc_maps(h);
  build_fused_map(h);
  *out = h;
  return PI_OK;
}

void pi_ffn_destroy(pi_ffn_t h) { delete h; }

pi_status pi_workspace_size(const pi_ffn_t *layers, int n_layers, int max_batch, size_t *bytes) {
  if (!layers || n_layers <= 0 || !bytes) return PI_ERR_INVALID_ARG;
  if (max_batch <= 0 || max_batch > kMaxBatch) return PI_ERR_UNSUPPORTED;
  for (int i = 0; i < n_layers; ++i)
    if (!layers[i]) return PI_ERR_INVALID_ARG;
  int dmax = 0, fmax = 0, rmax = 0;
  for (int i = 0; i < n_layers; ++i) {
    dmax = dmax > layers[i]->d.d_model ? dmax : layers[i]->d.d_model;
    fmax = fmax > layers[i]->d.d_ffn ? fmax : layers[i]->d.d_ffn;
    rmax = rmax > layers[i]->d.rank ? rmax : layers[i]->d.rank;
  }
  const int G = device_sm_count();
  if (G <= 0) return PI_ERR_CUDA;
  *bytes = ws_layout(dmax, fmax, rmax, max_batch, G).total;
  bool tc = false;
  for (int i = 0; i < n_layers; ++i) tc = tc || (layers[i]->tc_maps && max_batch >= tc_min_batch(layers[i]));
  if (tc) *bytes += tc_layout(dmax, fmax, rmax, G).total + 256;
  return PI_OK;
}

pi_status pi_workspace_init(void *ws, size_t ws_bytes, pi_stream_t stream) {
  if (!ws || ws_bytes == 0) return PI_ERR_INVALID_ARG;
  if (!aligned16(ws)) return PI_ERR_MISALIGNED;
  return cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream) == cudaSuccess ? PI_OK : PI_ERR_CUDA;
}

pi_status pi_predict(pi_ffn_t h, const void *u, int B, int32_t *idx, int32_t *count, void *ws, size_t ws_bytes,
                     pi_stream_t stream) {
  pi_status s = check_call(h, B);
  if (s != PI_OK) return s;
  if (!u || !idx || !count) return PI_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(idx) || !aligned16(count)) return PI_ERR_MISALIGNED;
  if (B == 0) return PI_OK;
  Ws w;
  const pi_ffn *L[1] = {h};
  if ((s = get_ws(L, 1, B, ws, ws_bytes, &w)) != PI_OK) return s;
  if (tc_ok(h, B) && !pred_batch_ok(h, B))
    return run_predict_tc(h, u, B, idx, h->d.d_ffn, count, w, (cudaStream_t)stream);
  return run_predict(h, u, B, idx, h->d.d_ffn, count, w, (cudaStream_t)stream);
}

pi_status pi_sparse_ffn(pi_ffn_t h, const void *u, int B, const int32_t *idx, const int32_t *count, float *y,
                        unsigned flags, void *ws, size_t ws_bytes, pi_stream_t stream) {
  pi_status s = check_call(h, B);
  if (s != PI_OK) return s;
  if (!u || !idx || !count || !y) return PI_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(idx) || !aligned16(count) || !aligned16(y)) return PI_ERR_MISALIGNED;
  if (flags & ~7u) return PI_ERR_INVALID_ARG;
  if (B == 0) return PI_OK;
  Ws w;
  const pi_ffn *L[1] = {h};
  if ((s = get_ws(L, 1, B, ws, ws_bytes, &w)) != PI_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if ((s = run_sets(h, idx, count, B, w, st)) != PI_OK) return s;
  if (tc_ok(h, B)) return run_ffn_tc(h, u, B, y, (flags & PI_FFN_ACCUMULATE) ? 1 : 0, false, w, st);
  return run_ffn(h, u, B, y, (flags & PI_FFN_ACCUMULATE) ? 1 : 0, flags, w, st);
}

pi_status pi_decode_ffn(pi_ffn_t h, const void *u, int B, float *y, int32_t *idx, int32_t *count, unsigned flags,
                        void *ws, size_t ws_bytes, pi_stream_t stream) {
  pi_status s = check_call(h, B);
  if (s != PI_OK) return s;
  if (!u || !y) return PI_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(y) || (idx && !aligned16(idx)) || (count && !aligned16(count)))
    return PI_ERR_MISALIGNED;
  if (flags & ~7u) return PI_ERR_INVALID_ARG;
  if (B == 0) return PI_OK;
  Ws w;
  const pi_ffn *L[1] = {h};
  if ((s = get_ws(L, 1, B, ws, ws_bytes, &w)) != PI_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int acc = (flags & PI_FFN_ACCUMULATE) ? 1 : 0;
  if (fused_ok(h, B, w.L.G)) return run_fused(h, u, y, 0, acc, idx, count, flags, w, st);
  if (tc_ok(h, B)) {
    // up to 8 tokens the batch predictor (fp16 predictor whatever the
    // weights) is the faster steps 1-2; it writes the mask and union words
    // the tensor-core FFN kernels read
    if (pred_batch_ok(h, B)) {
      if ((s = run_predict(h, u, B, idx, h->d.d_ffn, count, w, st)) != PI_OK) return s;
      return run_ffn_tc(h, u, B, y, acc, false, w, st);
    }
    if ((s = run_predict_tc(h, u, B, idx, h->d.d_ffn, count, w, st)) != PI_OK) return s;
    return run_ffn_tc(h, u, B, y, acc, true, w, st);
  }
  if ((s = run_predict(h, u, B, idx, h->d.d_ffn, count, w, st)) != PI_OK) return s;
  return run_ffn(h, u, B, y, acc, flags, w, st);
}

pi_status pi_decode_ffn_stack(const pi_ffn_t *layers, int L, float *x, int B, int32_t *idx_trace,
                              int32_t *count_trace, unsigned flags, void *ws, size_t ws_bytes, pi_stream_t stream) {
  if (!layers || L <= 0 || !x) return PI_ERR_INVALID_ARG;
  if (B < 0 || B > kMaxBatch) return PI_ERR_UNSUPPORTED;
  if (!aligned16(x) || (idx_trace && !aligned16(idx_trace)) || (count_trace && !aligned16(count_trace)))
    return PI_ERR_MISALIGNED;
  if (flags & ~6u) return PI_ERR_INVALID_ARG;
  int fmax = 0;
  for (int l = 0; l < L; ++l) {
    if (!layers[l]) return PI_ERR_INVALID_ARG;
    if (layers[l]->d.d_model != layers[0]->d.d_model) return PI_ERR_UNSUPPORTED;
    if (layers[l]->d.wtype == PI_W_F32) return PI_ERR_UNSUPPORTED;
    fmax = fmax > layers[l]->d.d_ffn ? fmax : layers[l]->d.d_ffn;
  }
  if (B == 0) return PI_OK;
  Ws w;
  pi_status s = get_ws(layers, L, B, ws, ws_bytes, &w);
  if (s != PI_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int d = layers[0]->d.d_model;
  for (int l = 0; l < L; ++l) {
    int32_t *idx = idx_trace ? idx_trace + (size_t)l * B * fmax : nullptr;
    int32_t *cnt = count_trace ? count_trace + (size_t)l * B : nullptr;
    if (fused_ok(layers[l], B, w.L.G)) {
      if ((s = run_fused(layers[l], x, x, 1, 0, idx, cnt, flags, w, st)) != PI_OK) return s;
      continue;
    }
    PI_CUDA(launch(pi::rmsnorm_kernel, dim3(B), dim3(256), st, (const float *)x, d, w.u()));
    if (tc_ok(layers[l], B)) {
      if (pred_batch_ok(layers[l], B)) {
        if ((s = run_predict(layers[l], w.u(), B, idx, fmax, cnt, w, st)) != PI_OK) return s;
        if ((s = run_ffn_tc(layers[l], w.u(), B, x, 1, false, w, st)) != PI_OK) return s;
      } else {
        if ((s = run_predict_tc(layers[l], w.u(), B, idx, fmax, cnt, w, st)) != PI_OK) return s;
        if ((s = run_ffn_tc(layers[l], w.u(), B, x, 1, true, w, st)) != PI_OK) return s;
      }
      continue;
    }
    if ((s = run_predict(layers[l], w.u(), B, idx, fmax, cnt, w, st)) != PI_OK) return s;
    if ((s = run_ffn(layers[l], w.u(), B, x, 1, flags, w, st)) != PI_OK) return s;
  }
  return PI_OK;
}

pi_status pi_decode_ffn_static(pi_ffn_t h, const void *u, float *y, int32_t *idx, int32_t *count, unsigned flags,
                               int *dev_status, pi_stream_t stream) {
  pi_status s = check_call(h, 1);
  if (s != PI_OK) return s;
  if (!u || !y) return PI_ERR_INVALID_ARG;
  if (!aligned16(u) || !aligned16(y) || (idx && !aligned16(idx)) || (count && !aligned16(count)) ||
      (reinterpret_cast<uintptr_t>(dev_status) & 3u))
    return PI_ERR_MISALIGNED;
  if (flags & ~7u) return PI_ERR_INVALID_ARG;
  void *base = nullptr;
  if ((s = static_scratch(&base)) != PI_OK) return s;
  const int G = device_sm_count();
  if (G <= 0) return PI_ERR_CUDA;
  Ws w;
  w.L = ws_layout(h->d.d_model, h->d.d_ffn, h->d.rank, 1, G);
  w.base = static_cast<char *>(base);
  if (w.L.total > PI_STATIC_SCRATCH_BYTES) return PI_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  // status word, union count and grid-barrier word must start at zero; the
  // kernels initialise the rest of the scratch they read
  PI_CUDA(cudaMemsetAsync(base, 0, 16, st));
  const int acc = (flags & PI_FFN_ACCUMULATE) ? 1 : 0;
  if (fused_ok(h, 1, G)) {
    s = run_fused(h, u, y, 0, acc, idx, count, flags, w, st);
  } else if ((s = run_predict(h, u, 1, idx, h->d.d_ffn, count, w, st)) == PI_OK) {
    s = run_ffn(h, u, 1, y, acc, flags, w, st);
  }
  if (s != PI_OK) return s;
  if (dev_status) PI_CUDA(cudaMemcpyAsync(dev_status, base, sizeof(int), cudaMemcpyDeviceToDevice, st));
  return PI_OK;
}

pi_status pi_debug_wait_fault(int withhold_row, unsigned limit_us) {
  if (withhold_row < -1) return PI_ERR_INVALID_ARG;
  if (withhold_row >= 0 && limit_us == 0) return PI_ERR_INVALID_ARG;
  g_wait_fault.withhold = withhold_row;
  g_wait_fault.limit_ns = (unsigned long long)limit_us * 1000ull;
  return PI_OK;
}

pi_status pi_get_device_status(void *ws, pi_stream_t stream, int *code) {
  if (!ws || !code) return PI_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return PI_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PI_ERR_CUDA;
  if (v != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return PI_ERR_CUDA;
  *code = v;
  return PI_OK;
}

const char *pi_status_string(pi_status s) {
  switch (s) {
  case PI_OK:
    return "ok";
  case PI_ERR_INVALID_ARG:
    return "invalid argument";
  case PI_ERR_UNSUPPORTED:
    return "unsupported shape or type";
  case PI_ERR_MISALIGNED:
    return "pointer not 16-byte aligned";
  case PI_ERR_CUDA:
    return "CUDA runtime error";
  case PI_ERR_TIMEOUT:
    return "device wait timed out";
  case PI_ERR_DEVICE_STATUS:
    return "device-side argument error";
  case PI_ERR_WORKSPACE:
    return "workspace missing or too small";
  }
  return "unknown status";
}

}  // extern "C"
