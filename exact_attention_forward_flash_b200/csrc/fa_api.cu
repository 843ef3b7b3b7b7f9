// fa_api.cu -- the C ABI of the attention forward library (declared in
// include/fa_b200.h): argument validation, TMA descriptor encoding, kernel
// selection and launch, the split-KV merge.  The forward kernels themselves
// are instantiated per width in fa_kern_w<W>.cu.  Nothing here allocates
// device memory or synchronises a stream (fa_check_device_error excepted, by
// its contract).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "fa_b200.h"
#include "fa_launch.cuh"

// The library's device error word (one per device): kernels record timeouts
// and broken input contracts here (see sm100_ptx.cuh); fa_check_device_error
// reads and clears it.
static __device__ unsigned g_fa_error;

namespace {
thread_local char g_msg[512] = "";
}  // namespace

namespace fab {

fa_status fail(fa_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

int num_sms(int dev) {
  static int cache[kMaxDev] = {0};
  if (dev < 0 || dev >= kMaxDev) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

}  // namespace fab

namespace fab {

// ---------------------------------------------------------------------------
// watchdog self-test: one thread waits, bounded by timeout_ns, on a fresh
// mbarrier that nothing ever arrives at, so the wait must give up, record the
// timeout code in the watchdog word and return (no trap, no endless loop).
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) fa_watchdog_selftest_kernel(unsigned *err,
                                                                  unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) (void)mbar_wait(smem_u32(&bar), 0u, err, timeout_ns);
}

// ---------------------------------------------------------------------------
// FMA-pipe exponential self-test: y = 2^x through ex2_poly2, the routine the
// softmax uses for part of its exponentials, element pairs per thread (an odd
// last element is paired with 0).  Lets a test measure its error on the GPU.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fa_selftest_exp2_fma_kernel(const float *__restrict__ x,
                                                                   float *__restrict__ y,
                                                                   long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const bool pair = i + 1 < n;
  float y0, y1;
  ex2_poly2(x[i], pair ? x[i + 1] : 0.f, y0, y1);
  y[i] = y0;
  if (pair) y[i + 1] = y1;
}

}  // namespace fab

namespace {

using namespace fab;

// ---------------------------------------------------------------------------
// driver entry point for tensor-map encoding (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Encoded maps are cached per host thread (a call encodes three, and the
// driver call dominates the host cost of small problems); the key is every
// input of the encoding.
struct MapKey {
  const void *base;
  long long tokens;
  int D, H, box_h, box_t, half;
  bool operator==(const MapKey &o) const {
    return base == o.base && tokens == o.tokens && D == o.D && H == o.H && box_h == o.box_h &&
           box_t == o.box_t && half == o.half;
  }
};
constexpr int kMapCache = 16;
struct MapCache {
  MapKey key[kMapCache];
  CUtensorMap map[kMapCache];
  bool used[kMapCache] = {};
  int next = 0;
};
thread_local MapCache g_maps;

fa_status encode_map(CUtensorMap *tm, const void *base, int D, int H, long long tokens, int box_h,
                     int box_t, bool half);

// 3-D map over a [tokens, heads, D] tensor of 16-bit elements with a box of
// {64 columns, box_h heads, box_t tokens}, 128-byte swizzle, zero fill.
int kernel_width(int D);

fa_status make_map(CUtensorMap *tm, const void *base, int D, int H, long long tokens, int box_h,
                   int box_t, bool half) {
  const MapKey k{base, tokens, D, H, box_h, box_t, half ? 1 : 0};
  for (int i = 0; i < kMapCache; ++i)
    if (g_maps.used[i] && g_maps.key[i] == k) {
      *tm = g_maps.map[i];
      return FA_OK;
    }
  fa_status s = encode_map(tm, base, D, H, tokens, box_h, box_t, half);
  if (s != FA_OK) return s;
  const int i = g_maps.next;
  g_maps.next = (i + 1) % kMapCache;
  g_maps.key[i] = k;
  g_maps.map[i] = *tm;
  g_maps.used[i] = true;
  return FA_OK;
}

fa_status encode_map(CUtensorMap *tm, const void *base, int D, int H, long long tokens, int box_h,
                     int box_t, bool half) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)tokens};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
  // head dims that are a multiple of 64: 64-column boxes, 128-byte swizzle;
  // narrow ones: 16-column boxes, 32-byte swizzle (the columns past D of the
  // last box read as zero)
  const bool narrow = kernel_width(D) % 64 != 0;
  cuuint32_t box[3] = {narrow ? 16u : 64u, (cuuint32_t)box_h, (cuuint32_t)box_t};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(tm, half ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  narrow ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return FA_OK;
}

// ---------------------------------------------------------------------------
// per-device state
// ---------------------------------------------------------------------------
// Device address of a __device__ variable, looked up with `dev` current (the
// caller passes the current device) and cached per device.
template <class T>
fa_status symbol_address(T &sym, int dev, void **cache, std::mutex &mu, void **addr,
                         const char *what) {
  if (dev < 0 || dev >= kMaxDev) return fail(FA_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == nullptr) {
    void *ptr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&ptr, sym);
    if (e != cudaSuccess || ptr == nullptr)
      return fail(FA_ERR_CUDA, "looking up %s: %s", what, cudaGetErrorString(e));
    cache[dev] = ptr;
  }
  *addr = cache[dev];
  return FA_OK;
}

fa_status error_word(int dev, unsigned **addr) {
  static std::mutex mu;
  static void *cache[kMaxDev] = {nullptr};
  void *a = nullptr;
  fa_status s = symbol_address(g_fa_error, dev, cache, mu, &a, "the device error word");
  *addr = static_cast<unsigned *>(a);
  return s;
}

// The current device and its error word.
fa_status current_device(int *dev, unsigned **err) {
  if (cudaGetDevice(dev) != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice failed");
  return error_word(*dev, err);
}

// The kernel of width w and kind k.
fa_status launch_width(int w, Kind k, FwdParams &p, int dev, cudaStream_t st, bool half,
                       bool mods) {
  switch (w) {
    case 16: return launch_w16(k, p, dev, st, half, mods);
    case 32: return launch_w32(k, p, dev, st, half, mods);
    case 48: return launch_w48(k, p, dev, st, half, mods);
    case 64: return launch_w64(k, p, dev, st, half, mods);
    case 80: return launch_w80(k, p, dev, st, half, mods);
    case 96: return launch_w96(k, p, dev, st, half, mods);
    case 128: return launch_w128(k, p, dev, st, half, mods);
    default: return launch_w256(k, p, dev, st, half, mods);
  }
}

// the modifier kernels serve a left window bound or a soft-cap (the plain
// ones serve causal masking and any right window bound)
bool uses_mods(const FwdParams &p) { return p.wl >= 0 || p.cap_a > 0.f; }

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr unsigned long long kTimeoutNs = 4000000000ull;  // 4 s per wait

struct Common {
  const void *q, *k, *v;
  void *out;
  float *lse;
  const int *cu_q, *cu_k, *seqused_k;
  const void *rel_bias;
  int R, B, Sq, Sk, Hq, Hkv, D, total_q, total_k, max_q;
  fa_dtype dt;
  int causal;
  float scale;
  bool varlen;
  // modifiers (fa_mods): window bounds (< 0: none), soft-cap (0: off)
  int window_left = -1, window_right = -1;
  float softcap = 0.f;
  // key shard: per-batch count of the sequence's keys after the ones given
  const int *k_after = nullptr;
};

void apply_mods(Common &c, const fa_mods *m) {
  if (m == nullptr) return;
  c.window_left = m->window_left;
  c.window_right = m->window_right;
  c.softcap = m->softcap;
}

// Head dims: every multiple of 8 from 16 to 256.  Each runs in the kernel of
// the next width up; the tensors keep their own D (row pitch D), the columns
// past D read as zeros (the loads fill them) and are never stored.  Widths:
// 64, 128 and 256 with 64-column chunks and a 128-byte swizzle; 16, 32, 48,
// 80 and 96 with 16-column chunks and a 32-byte swizzle.
bool head_dim_served(int D) { return D % 8 == 0 && D >= 16 && D <= 256; }

int kernel_width(int D) {
  if (D == 64 || D == 128 || D == 256) return D;
  if (D <= 48) return (D + 15) / 16 * 16;  // 16, 32, 48
  if (D <= 80) return 80;                  // 56, 72, 80
  if (D <= 96) return 96;                  // 88, 96
  if (D <= 128) return 128;                // 104 .. 120
  return 256;                              // 136 .. 248
}

fa_status validate(const Common &c) {
  if (c.dt != FA_BF16 && c.dt != FA_FP16) return fail(FA_ERR_INVALID, "dtype must be bf16 or fp16");
  if (c.B < 0 || c.Hq <= 0 || c.Hkv <= 0 || c.D <= 0)
    return fail(FA_ERR_INVALID, "B must be >= 0 and Hq, Hkv, D > 0");
  if (c.Hq % c.Hkv != 0) return fail(FA_ERR_INVALID, "Hq (%d) must be a multiple of Hkv (%d)", c.Hq, c.Hkv);
  if (!head_dim_served(c.D))
    return fail(FA_ERR_UNSUPPORTED, "head_dim %d not served (multiples of 8 from 16 to 256)", c.D);
  if (!c.varlen && (c.Sq < 0 || c.Sk < 0)) return fail(FA_ERR_INVALID, "Sq, Sk must be >= 0");
  if (c.varlen && (c.total_q < 0 || c.total_k < 0 || c.max_q < 0))
    return fail(FA_ERR_INVALID, "total_q, total_k, max_seqlen_q must be >= 0");
  if (c.rel_bias != nullptr) {
    if (c.R <= 0 || c.R % 128 != 0)
      return fail(FA_ERR_INVALID, "rel_extent (%d) must be a positive multiple of 128", c.R);
    if (!aligned16(c.rel_bias)) return fail(FA_ERR_INVALID, "rel_bias must be 16-byte aligned");
    // B * Sq * Hq * rel_extent elements of 2 bytes; the product is taken in
    // 128 bits (B * Sq alone may reach 2^62 before the token-count rule)
    const unsigned __int128 tqb =
        c.varlen ? (unsigned __int128)c.total_q : (unsigned __int128)c.B * (unsigned)c.Sq;
    if (tqb * (unsigned)c.Hq * (unsigned)c.R * 2u >= ((unsigned __int128)64 << 30))
      return fail(FA_ERR_UNSUPPORTED, "rel_bias larger than 64 GiB");
  }
  if (!std::isfinite(c.scale)) return fail(FA_ERR_INVALID, "softmax_scale must be finite");
  if (!std::isfinite(c.softcap) || c.softcap < 0.f)
    return fail(FA_ERR_INVALID, "softcap must be finite and >= 0");
  const long long tq = c.varlen ? c.total_q : (long long)c.B * c.Sq;
  const long long tk = c.varlen ? c.total_k : (long long)c.B * c.Sk;
  if (tq > 0x7fffffffLL || tk > 0x7fffffffLL || tq * c.Hq > (1LL << 40))
    return fail(FA_ERR_UNSUPPORTED, "problem too large for 32-bit token indices");
  if (tq > 0) {
    if (!c.q || !c.out) return fail(FA_ERR_INVALID, "q and out must not be NULL");
    if (!aligned16(c.q) || !aligned16(c.out)) return fail(FA_ERR_INVALID, "q/out must be 16-byte aligned");
    if (tk > 0) {
      if (!c.k || !c.v) return fail(FA_ERR_INVALID, "k and v must not be NULL");
      if (!aligned16(c.k) || !aligned16(c.v)) return fail(FA_ERR_INVALID, "k/v must be 16-byte aligned");
    }
  }
  if (c.varlen && c.B > 0 && (!c.cu_q || !c.cu_k))
    return fail(FA_ERR_INVALID, "cu_seqlens_q and cu_seqlens_k must not be NULL");
  return FA_OK;
}

// Query heads packed per tile: all heads of a K/V group when that divides 128.
// (a divisor of 128, hence a power of two)
int pack_factor(int G) { return (G >= 1 && G <= 128 && 128 % G == 0) ? G : 1; }

fa_status fill_params(const Common &c, FwdParams &p, int nq, int bn, int num_splits,
                      int split_keys) {
  std::memset(&p, 0, sizeof(p));
  const bool half = c.dt == FA_FP16;
  const int G = c.Hq / c.Hkv;
  const int P = pack_factor(G);
  const long long tq = c.varlen ? c.total_q : (long long)c.B * c.Sq;
  const long long tk = c.varlen ? c.total_k : (long long)c.B * c.Sk;
  fa_status s;
  if ((s = make_map(&p.tm_q, c.q, c.D, c.Hq, tq, P, kBM / P, half)) != FA_OK) return s;
  // With no keys at all every unit is empty and K/V are never read; the maps
  // then describe one token of q (which holds at least Hkv * D elements).
  const void *kb = tk > 0 ? c.k : c.q;
  const void *vb = tk > 0 ? c.v : c.q;
  const long long tkm = tk > 0 ? tk : 1;
  if ((s = make_map(&p.tm_k, kb, c.D, c.Hkv, tkm, 1, bn, half)) != FA_OK) return s;
  if ((s = make_map(&p.tm_v, vb, c.D, c.Hkv, tkm, 1, bn, half)) != FA_OK) return s;
  p.out = c.out;
  p.lse = c.lse;
  p.cu_q = c.varlen ? c.cu_q : nullptr;
  p.cu_k = c.varlen ? c.cu_k : nullptr;
  p.seqused_k = c.seqused_k;
  p.k_after = c.k_after;
  p.rel_bias = static_cast<const uint16_t *>(c.rel_bias);
  p.R = c.rel_bias ? c.R : 0;
  p.d_out = c.D;
  // 32-byte epilogue stores: the output base and every row 32-byte aligned
  // (rows of 16-bit outputs hold D * 2 bytes, fp32 partials D * 4)
  p.st32 = ((reinterpret_cast<uintptr_t>(c.out) & 31) == 0 && c.D % 16 == 0) ? 1 : 0;
  p.B = c.B;
  p.Sq = c.Sq;
  p.Sk = c.Sk;
  p.Hq = c.Hq;
  p.Hkv = c.Hkv;
  p.G = G;
  p.P = P;
  p.lgP = 0;
  while ((1 << p.lgP) < P) ++p.lgP;
  p.n_groups = c.Hq / P;
  p.total_q = (int)tq;
  p.total_k = (int)tk;
  const int max_q = c.varlen ? c.max_q : c.Sq;
  p.max_q = max_q;
  const long long rows = (long long)max_q * P;
  p.n_mblk = (int)std::max<long long>(1, (rows + (long long)nq * kBM - 1) / ((long long)nq * kBM));
  p.num_splits = num_splits;
  p.split_keys = split_keys;
  p.causal = c.causal ? 1 : 0;
  p.m_major = c.causal ? 1 : 0;
  p.lse_dense = c.varlen ? 0 : 1;
  const long long units = (long long)c.B * p.n_groups * p.n_mblk * num_splits;
  if (units > 0x7fffffffLL) return fail(FA_ERR_UNSUPPORTED, "too many work units");
  p.num_units = (int)units;
  const float scale = c.scale > 0.f ? c.scale : 1.0f / std::sqrt((float)c.D);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.inv_scale = 1.0f / scale;
  p.thr_raw = 8.0f / p.scale_log2;
  p.wl = c.window_left < 0 ? -1 : c.window_left;
  p.wr = c.causal ? 0 : (c.window_right < 0 ? -1 : c.window_right);
  if (c.softcap > 0.f) {
    p.cap_a = c.softcap / scale;  // raw-score units
    p.cap_b = scale / c.softcap;
  }
  p.timeout_ns = kTimeoutNs;
  return FA_OK;
}

fa_status run_fwd(const Common &c, cudaStream_t st) {
  fa_status s = validate(c);
  if (s != FA_OK) return s;
  const long long tq = c.varlen ? c.total_q : (long long)c.B * c.Sq;
  if (tq == 0 || c.B == 0) return FA_OK;  // nothing to compute
  int dev = 0;
  unsigned *err = nullptr;
  if ((s = current_device(&dev, &err)) != FA_OK) return s;
  FwdParams p;
  // width <= 128: two Q tiles per CTA, 128-key tiles.  Width 256: units of
  // two Q tiles on a CTA pair (one tile per SM) with 128-key tiles, of which
  // each CTA loads 64 keys of K and 128 dims of V -- when there is more than
  // one wave of pairs; a problem of at most one wave runs one Q tile per CTA
  // with 64-key tiles, whose shorter start-up and teardown (no cluster
  // barriers) weigh more there than the pair's faster key loop.
  const int w = kernel_width(c.D);
  if ((s = fill_params(c, p, 2, 128, 1, 0x7fffffff)) != FA_OK) return s;
  if (p.num_units == 0) return FA_OK;
  const bool half = c.dt == FA_FP16;
  const bool mods = uses_mods(p);
  Kind kind = Kind::kThroughput;
  if (w == 256 && p.num_units > num_sms(dev) / 2) {
    // K is loaded in halves of 64 keys
    const long long tk = c.varlen ? c.total_k : (long long)c.B * c.Sk;
    if ((s = make_map(&p.tm_k, tk > 0 ? c.k : c.q, c.D, c.Hkv, tk > 0 ? tk : 1, 1, 64, half)) != FA_OK)
      return s;
    kind = Kind::kPair;
  } else if (w == 256) {
    if ((s = fill_params(c, p, 1, 64, 1, 0x7fffffff)) != FA_OK) return s;
  } else if (p.num_units < num_sms(dev)) {
    // fewer two-tile units than SMs: one tile per CTA, twice the units
    if ((s = fill_params(c, p, 1, 128, 1, 0x7fffffff)) != FA_OK) return s;
    kind = Kind::kLatency;
  } else if (w <= 96) {
    // Widths 16 to 96 take three Q tiles per CTA (no relative bias; 64-key
    // tiles from width 48 up, where three 128-key S buffers and O tiles would
    // not fit in tensor memory): each tile runs about 1.1x faster than with two,
    // since the softmax of three tiles hides more of each other's latency;
    // the unit count drops by a third, so the choice compares whole waves.
    kind = Kind::kTwoTile;
    if (c.rel_bias == nullptr) {
      const long long sms = num_sms(dev), w2 = (p.num_units + sms - 1) / sms;
      FwdParams p3;
      if ((s = fill_params(c, p3, 3, w <= 32 ? 128 : 64, 1, 0x7fffffff)) != FA_OK) return s;
      const long long w3 = (p3.num_units + sms - 1) / sms;
      if (w3 * 3 * 10 <= w2 * 2 * 11) {
        p = p3;
        kind = Kind::kThroughput;
      }
    }
  }
  p.err = err;
  return launch_width(w, kind, p, dev, st, half, mods);
}

template <int D, bool HALF, bool F32OUT>
fa_status launch_combine(const float *o_part, const float *lse_part, int ns, long long rows,
                         void *out, float *lse, int Hq, int Sq, int total_q, int lse_dense,
                         cudaStream_t st) {
  const int warps = 8;
  const long long blocks = (rows + warps - 1) / warps;
  if (blocks > 0x7fffffffLL) return fail(FA_ERR_UNSUPPORTED, "too many rows");
  fa_combine_kernel<D, HALF, F32OUT><<<(unsigned)blocks, warps * 32, 0, st>>>(
      o_part, lse_part, ns, rows, out, lse, Hq, Sq, total_q, lse_dense);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

// Merge ns partials of `rows` packed rows of a dense [B, Sq, Hq] problem:
// into out (input dtype) and lse [B, Hq, Sq], or, with f32out, into one
// fp32 partial (out [rows][D], lse [rows]).
fa_status combine(int D, bool half, bool f32out, const float *o_part, const float *lse_part,
                  int ns, long long rows, void *out, float *lse, int Hq, int Sq, int B,
                  cudaStream_t st) {
  const int tq = B * Sq;
#define FA_COMBINE(DD)                                                                      \
  if (f32out)                                                                               \
    return launch_combine<DD, false, true>(o_part, lse_part, ns, rows, out, lse, Hq, Sq, tq, \
                                           1, st);                                          \
  return half ? launch_combine<DD, true, false>(o_part, lse_part, ns, rows, out, lse, Hq, Sq, \
                                                tq, 1, st)                                   \
              : launch_combine<DD, false, false>(o_part, lse_part, ns, rows, out, lse, Hq,  \
                                                 Sq, tq, 1, st);
  if (D % 64 != 0) {
    const int warps = 8;
    const long long blocks = (rows + warps - 1) / warps;
    if (blocks > 0x7fffffffLL) return fail(FA_ERR_UNSUPPORTED, "too many rows");
    if (f32out)
      fa_combine_narrow_kernel<false, true><<<(unsigned)blocks, warps * 32, 0, st>>>(
          o_part, lse_part, ns, rows, D, out, lse, Hq, Sq);
    else if (half)
      fa_combine_narrow_kernel<true, false><<<(unsigned)blocks, warps * 32, 0, st>>>(
          o_part, lse_part, ns, rows, D, out, lse, Hq, Sq);
    else
      fa_combine_narrow_kernel<false, false><<<(unsigned)blocks, warps * 32, 0, st>>>(
          o_part, lse_part, ns, rows, D, out, lse, Hq, Sq);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "combine launch: %s", cudaGetErrorString(e));
    return FA_OK;
  }
  if (D == 64) { FA_COMBINE(64) }
  if (D == 128) { FA_COMBINE(128) }
  FA_COMBINE(256)
#undef FA_COMBINE
}

int splitkv_bn(int D) { return kernel_width(D) == 256 ? 64 : 128; }

// The split count a split-KV call launches and the keys of each split
// (whole key tiles): num_splits (0 = the default for this device) capped at
// one split per key tile, then reduced to the splits that the rounded split
// length actually needs.
struct SplitPlan {
  int ns, split_keys;
};

SplitPlan plan_splits(int B, int Sq, int Sk, int Hq, int Hkv, int D, int num_splits, int n_sms) {
  const int bn = splitkv_bn(D);
  int ns = num_splits > 0 ? num_splits : fa_splitkv_default_splits(B, Sq, Sk, Hq, Hkv, D, n_sms);
  const long long tiles = std::max<long long>(1, ((long long)Sk + bn - 1) / bn);
  if (ns > tiles) ns = (int)tiles;
  if (ns < 1) ns = 1;
  const int split_keys = (int)(((tiles + ns - 1) / ns) * bn);
  ns = (int)std::max<long long>(1, ((long long)Sk + split_keys - 1) / split_keys);
  return {ns, split_keys};
}

// Split-KV forward of a dense problem: the keys are cut into num_splits
// ranges whose normalised fp32 partials go to the workspace and are merged
// by LSE into c.out / c.lse, or, with to_partial, into one fp32 partial
// (c.out as float [B*Sq*Hq][D], c.lse as float [B*Sq*Hq]).  A single split
// writes a partial in place and needs no workspace.
fa_status run_splitkv(const Common &c, int num_splits, void *workspace, size_t workspace_bytes,
                      bool to_partial, cudaStream_t st) {
  fa_status s = validate(c);
  if (s != FA_OK) return s;
  if (num_splits < 0) return fail(FA_ERR_INVALID, "num_splits must be >= 0");
  const int B = c.B, Sq = c.Sq, Sk = c.Sk, Hq = c.Hq, D = c.D;
  if ((long long)B * Sq == 0) return FA_OK;
  int dev = 0;
  unsigned *err = nullptr;
  if ((s = current_device(&dev, &err)) != FA_OK) return s;
  if (Sk == 0 && !to_partial) return run_fwd(c, st);  // nothing to split
  const int bn = splitkv_bn(D);
  const SplitPlan sp = plan_splits(B, Sq, Sk, Hq, c.Hkv, D, num_splits, num_sms(dev));
  const int ns = sp.ns;
  const long long rows = (long long)B * Sq * Hq;
  const bool direct = to_partial && ns == 1;
  if (!direct) {
    const size_t need = fa_splitkv_workspace_bytes(B, Sq, Hq, D, ns);
    if (workspace == nullptr || workspace_bytes < need)
      return fail(FA_ERR_WORKSPACE, "workspace of %zu bytes needed, %zu given", need,
                  workspace_bytes);
    if (!aligned16(workspace)) return fail(FA_ERR_INVALID, "workspace must be 16-byte aligned");
  }
  FwdParams p;
  if ((s = fill_params(c, p, 1, bn, ns, sp.split_keys)) != FA_OK) return s;
  p.err = err;
  if (direct) {
    p.o_part = static_cast<float *>(c.out);
    p.lse_part = c.lse;
  } else {
    p.o_part = static_cast<float *>(workspace);
    p.lse_part = p.o_part + (size_t)ns * rows * D;
  }
  // fp32 partial rows hold D * 4 bytes (a multiple of 32): only the base counts
  p.st32 = (reinterpret_cast<uintptr_t>(p.o_part) & 31) == 0 ? 1 : 0;
  const bool half = c.dt == FA_FP16;
  s = launch_width(kernel_width(D), Kind::kPartial, p, dev, st, half, uses_mods(p));
  if (s != FA_OK || direct) return s;
  return combine(D, half, to_partial, p.o_part, p.lse_part, ns, rows, c.out, c.lse, Hq, Sq, B,
                 st);
}

}  // namespace

extern "C" {

const char *fa_status_string(fa_status s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID: return "FA_ERR_INVALID";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_DEVICE_TIMEOUT: return "FA_ERR_DEVICE_TIMEOUT";
  }
  return "FA_ERR_UNKNOWN";
}

const char *fa_last_error_message(void) { return g_msg; }

const char *fa_version(void) { return "fa_b200 0.1 (sm_100a)"; }

fa_status fa_fwd_ex(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                    int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt, int causal,
                    float softmax_scale, const int *seqused_k, const void *rel_bias,
                    int rel_extent, const fa_mods *mods, void *stream) {
  g_msg[0] = 0;
  Common c{q, k, v, out, lse, nullptr, nullptr, seqused_k, rel_bias, rel_extent, B, Sq, Sk,
           Hq, Hkv, D, 0, 0, 0, dt, causal, softmax_scale, false};
  apply_mods(c, mods);
  return run_fwd(c, static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd(const void *q, const void *k, const void *v, void *out, float *lse, int B,
                 int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt, int causal,
                 float softmax_scale, const int *seqused_k, const void *rel_bias, int rel_extent,
                 void *stream) {
  return fa_fwd_ex(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, causal, softmax_scale,
                   seqused_k, rel_bias, rel_extent, nullptr, stream);
}

fa_status fa_fwd_varlen_ex(const void *q, const void *k, const void *v, void *out, float *lse,
                           const int *cu_seqlens_q, const int *cu_seqlens_k,
                           const int *seqused_k, int B, int max_seqlen_q, int max_seqlen_k,
                           int total_q, int total_k, int Hq, int Hkv, int D, fa_dtype dt,
                           int causal, float softmax_scale, const void *rel_bias,
                           int rel_extent, const fa_mods *mods, void *stream) {
  g_msg[0] = 0;
  (void)max_seqlen_k;
  Common c{q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, seqused_k, rel_bias, rel_extent, B,
           0, 0, Hq, Hkv, D, total_q, total_k, max_seqlen_q, dt, causal, softmax_scale, true};
  apply_mods(c, mods);
  return run_fwd(c, static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_varlen(const void *q, const void *k, const void *v, void *out, float *lse,
                        const int *cu_seqlens_q, const int *cu_seqlens_k, const int *seqused_k,
                        int B, int max_seqlen_q, int max_seqlen_k, int total_q, int total_k,
                        int Hq, int Hkv, int D, fa_dtype dt, int causal, float softmax_scale,
                        const void *rel_bias, int rel_extent, void *stream) {
  return fa_fwd_varlen_ex(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, seqused_k, B,
                          max_seqlen_q, max_seqlen_k, total_q, total_k, Hq, Hkv, D, dt, causal,
                          softmax_scale, rel_bias, rel_extent, nullptr, stream);
}

size_t fa_splitkv_workspace_bytes(int B, int Sq, int Hq, int D, int num_splits) {
  if (B <= 0 || Sq <= 0 || Hq <= 0 || D <= 0 || num_splits <= 0) return 0;
  const size_t rows = (size_t)B * Sq * Hq;
  size_t bytes = (size_t)num_splits * rows * (size_t)(D + 1) * sizeof(float);
  return (bytes + 255) & ~(size_t)255;
}

int fa_splitkv_default_splits(int B, int Sq, int Sk, int Hq, int Hkv, int D, int n_sms) {
  if (B <= 0 || Sq <= 0 || Sk <= 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv) return 1;
  if (n_sms <= 0) n_sms = 148;
  const int bn = splitkv_bn(D);
  const int P = pack_factor(Hq / Hkv);
  const long long mblk = ((long long)Sq * P + kBM - 1) / kBM;
  const long long base = (long long)B * (Hq / P) * mblk;  // units without splitting
  // splits of at least 8 key tiles keep a decode streaming; a short call
  // whose units cover under a quarter of the SMs trades that for latency and
  // splits down to 2 tiles
  const int min_tiles = base * 4 >= n_sms ? 8 : 2;
  const long long max_by_len =
      std::max<long long>(1, ((long long)Sk + min_tiles * bn - 1) / (min_tiles * bn));
  if (base >= 4LL * n_sms) return 1;
  // enough units for about 16 per SM, in whole waves where possible
  long long ns = (16LL * n_sms + base - 1) / base;
  ns = std::min(ns, max_by_len);
  ns = std::min<long long>(ns, 256);
  return (int)std::max<long long>(1, ns);
}

fa_status fa_fwd_splitkv(const void *q, const void *k, const void *v, void *out, float *lse,
                         int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt, int causal,
                         float softmax_scale, const int *seqused_k, const void *rel_bias,
                         int rel_extent, int num_splits, void *workspace, size_t workspace_bytes,
                         void *stream) {
  return fa_fwd_splitkv_ex(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, causal, softmax_scale,
                           seqused_k, rel_bias, rel_extent, num_splits, workspace,
                           workspace_bytes, nullptr, stream);
}

fa_status fa_fwd_splitkv_ex(const void *q, const void *k, const void *v, void *out, float *lse,
                            int B, int Sq, int Sk, int Hq, int Hkv, int D, fa_dtype dt,
                            int causal, float softmax_scale, const int *seqused_k,
                            const void *rel_bias, int rel_extent, int num_splits,
                            void *workspace, size_t workspace_bytes, const fa_mods *mods,
                            void *stream) {
  g_msg[0] = 0;
  Common c{q, k, v, out, lse, nullptr, nullptr, seqused_k, rel_bias, rel_extent, B, Sq, Sk,
           Hq, Hkv, D, 0, 0, 0, dt, causal, softmax_scale, false};
  apply_mods(c, mods);
  return run_splitkv(c, num_splits, workspace, workspace_bytes, false,
                     static_cast<cudaStream_t>(stream));
}

fa_status fa_fwd_shard_partial(const void *q, const void *k, const void *v, float *o_part,
                               float *lse_part, int B, int Sq, int Sk, int Hq, int Hkv, int D,
                               fa_dtype dt, int causal, float softmax_scale,
                               const int *seqused_k, const int *k_after, const void *rel_bias,
                               int rel_extent, const fa_mods *mods, int num_splits,
                               void *workspace, size_t workspace_bytes, void *stream) {
  g_msg[0] = 0;
  if (lse_part == nullptr && (long long)B * Sq > 0)
    return fail(FA_ERR_INVALID, "lse_part must not be NULL");
  Common c{q, k, v, o_part, lse_part, nullptr, nullptr, seqused_k, rel_bias, rel_extent, B,
           Sq, Sk, Hq, Hkv, D, 0, 0, 0, dt, causal, softmax_scale, false};
  apply_mods(c, mods);
  c.k_after = k_after;
  return run_splitkv(c, num_splits, workspace, workspace_bytes, true,
                     static_cast<cudaStream_t>(stream));
}

fa_status fa_combine_partials(const float *o_parts, const float *lse_parts, int n_parts, int B,
                              int Sq, int Hq, int D, fa_dtype dt, void *out, float *lse,
                              void *stream) {
  g_msg[0] = 0;
  if (dt != FA_BF16 && dt != FA_FP16) return fail(FA_ERR_INVALID, "dtype must be bf16 or fp16");
  if (B < 0 || Sq < 0 || Hq <= 0) return fail(FA_ERR_INVALID, "B, Sq must be >= 0 and Hq > 0");
  if (!head_dim_served(D))
    return fail(FA_ERR_UNSUPPORTED, "head_dim %d not served (multiples of 8 from 16 to 256)", D);
  if (n_parts < 1) return fail(FA_ERR_INVALID, "n_parts must be >= 1");
  const long long rows = (long long)B * Sq * Hq;
  if (rows == 0) return FA_OK;
  if ((long long)B * Sq > 0x7fffffffLL) return fail(FA_ERR_UNSUPPORTED, "too many tokens");
  if (!o_parts || !lse_parts || !out) return fail(FA_ERR_INVALID, "o_parts, lse_parts and out must not be NULL");
  if (!aligned16(o_parts) || !aligned16(out)) return fail(FA_ERR_INVALID, "o_parts/out must be 16-byte aligned");
  return combine(D, dt == FA_FP16, false, o_parts, lse_parts, n_parts, rows, out, lse, Hq, Sq, B,
                 static_cast<cudaStream_t>(stream));
}

fa_status fa_watchdog_selftest(unsigned long long timeout_ns, void *stream) {
  g_msg[0] = 0;
  if (timeout_ns < 1000000ull || timeout_ns > 1000000000ull)
    return fail(FA_ERR_INVALID, "timeout_ns must be within [1 ms, 1 s]");
  int dev = 0;
  unsigned *err = nullptr;
  fa_status s = current_device(&dev, &err);
  if (s != FA_OK) return s;
  fab::fa_watchdog_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(err, timeout_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

fa_status fa_selftest_exp2_fma(const float *x, float *y, long long n, void *stream) {
  g_msg[0] = 0;
  if (n < 0) return fail(FA_ERR_INVALID, "n must be >= 0");
  if (n == 0) return FA_OK;
  if (x == nullptr || y == nullptr) return fail(FA_ERR_INVALID, "x and y must not be NULL");
  const long long threads = 256, pairs = (n + 1) / 2;
  const long long blocks = (pairs + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return fail(FA_ERR_UNSUPPORTED, "n too large");
  fab::fa_selftest_exp2_fma_kernel<<<(unsigned)blocks, (unsigned)threads, 0,
                                     static_cast<cudaStream_t>(stream)>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "self-test launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

fa_status fa_check_device_error(int *code, int clear) {
  unsigned v = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaDeviceSynchronize: %s", cudaGetErrorString(e));
  e = cudaMemcpyFromSymbol(&v, g_fa_error, sizeof(v));
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "reading the error word: %s", cudaGetErrorString(e));
  if (code) *code = (int)v;
  if (clear && v) {
    unsigned z = 0;
    e = cudaMemcpyToSymbol(g_fa_error, &z, sizeof(z));
    if (e != cudaSuccess) return fail(FA_ERR_CUDA, "clearing the error word: %s", cudaGetErrorString(e));
  }
  if (v & fab::kErrTimeout) return FA_ERR_DEVICE_TIMEOUT;
  if (v & fab::kErrInput) return FA_ERR_DEVICE_INPUT;
  return FA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Split-KV forward without any allocation by the caller or the library.
//
// The split partials live in one file-scope device array instead of a
// caller-provided workspace.  Its size is fixed at build time
// (FA_SPLITKV_STATIC_SCRATCH_BYTES) and it is held by every GPU that loads
// this library until the process exits.  Host code only sees a stand-in for
// the array's name, so its device address is looked up once per device (with
// that device current) by the first call made on that device.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_splitkv_scratch[FA_SPLITKV_STATIC_SCRATCH_BYTES];

namespace {

fa_status splitkv_scratch_address(int dev, void **addr) {
  static std::mutex mu;
  static void *cache[kMaxDev] = {nullptr};
  return symbol_address(g_splitkv_scratch, dev, cache, mu, addr, "the static split-KV scratch");
}

}  // namespace

extern "C" fa_status fa_fwd_splitkv_static(const void *q, const void *k, const void *v, void *out,
                                           float *lse, int B, int Sq, int Sk, int Hq, int Hkv,
                                           int D, fa_dtype dt, int causal, float softmax_scale,
                                           const int *seqused_k, const void *rel_bias,
                                           int rel_extent, int num_splits, void *stream) {
  g_msg[0] = 0;
  if (num_splits < 0) return fail(FA_ERR_INVALID, "num_splits must be >= 0");
  // the scratch address belongs to the device that is current for this call
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice failed");
  if ((long long)B * Sq > 0 && Sk > 0 && Hq > 0 && Hkv > 0 && Hq % Hkv == 0 && D > 0) {
    // the split count fa_fwd_splitkv will launch, and the scratch it needs
    const SplitPlan sp = plan_splits(B, Sq, Sk, Hq, Hkv, D, num_splits, num_sms(dev));
    const size_t need = fa_splitkv_workspace_bytes(B, Sq, Hq, D, sp.ns);
    if (need > (size_t)FA_SPLITKV_STATIC_SCRATCH_BYTES)
      return fail(FA_ERR_WORKSPACE,
                  "split-KV partials need %zu bytes, more than the %zu-byte static scratch "
                  "(use fa_fwd_splitkv with a workspace, or fewer splits)",
                  need, (size_t)FA_SPLITKV_STATIC_SCRATCH_BYTES);
  }
  void *scratch = nullptr;
  fa_status s = splitkv_scratch_address(dev, &scratch);
  if (s != FA_OK) return s;
  return fa_fwd_splitkv(q, k, v, out, lse, B, Sq, Sk, Hq, Hkv, D, dt, causal, softmax_scale,
                        seqused_k, rel_bias, rel_extent, num_splits, scratch,
                        (size_t)FA_SPLITKV_STATIC_SCRATCH_BYTES, stream);
}
