// fa_launch.cuh -- host-side launch of the forward kernel configurations,
// shared by the library's translation units: fa_api.cu holds the C ABI
// (validation, tensor maps, split planning, the merge), and one
// fa_kern_w<W>.cu per kernel width instantiates that width's kernels, so
// that the widths compile in parallel.
#pragma once

#include <cuda_runtime.h>

#include <algorithm>

#include "fa_b200.h"
#include "fa_fwd_kernel.cuh"

namespace fab {

constexpr int kMaxDev = 64;

// Records a message for fa_last_error_message() and returns s.
fa_status fail(fa_status s, const char *fmt, ...);

// Streaming multiprocessors of device dev (cached).
int num_sms(int dev);

// The kernel shapes of a width: several Q tiles per CTA with a single S
// buffer each (throughput: two tiles, three at widths 16 to 96), one Q tile
// with a double-buffered S (calls with fewer two-tile units than SMs), the
// split-KV partial kernel, (width 256) the CTA-pair kernel whose units of 256
// rows span two SMs, and two tiles per CTA where the throughput kernel takes
// three (widths 16 to 96 with a relative bias, or when three-tile units
// would leave more of the last wave idle).
enum class Kind { kThroughput, kLatency, kPartial, kPair, kTwoTile };

template <class C>
fa_status launch_fwd(FwdParams &p, int dev, cudaStream_t st) {
  static bool configured[kMaxDev] = {false};
  if (dev >= 0 && dev < kMaxDev && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(fa_fwd_kernel<C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess)
      return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    configured[dev] = true;
  }
  // causal problems with few enough sequences use the compact schedule
  p.compact = (p.m_major && p.B >= 1 && p.B <= C::kMaxSchedB) ? 1 : 0;
  const int grid = std::min(p.num_units, num_sms(dev));
  fa_fwd_kernel<C><<<grid, C::kThreads, C::kSmemBytes, st>>>(p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "kernel launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

// one of the four variants (bf16 / fp16, modifiers off / on) of a configuration
template <template <bool, bool> class Cfg>
fa_status launch_variant(FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (half) return mods ? launch_fwd<Cfg<true, true>>(p, dev, st) : launch_fwd<Cfg<true, false>>(p, dev, st);
  return mods ? launch_fwd<Cfg<false, true>>(p, dev, st) : launch_fwd<Cfg<false, false>>(p, dev, st);
}

// The three kinds of one width, given as configuration templates.
template <template <bool, bool> class Fwd, template <bool, bool> class Lat,
          template <bool, bool> class Spl>
fa_status launch_kind(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  switch (k) {
    case Kind::kThroughput:
    case Kind::kTwoTile: return launch_variant<Fwd>(p, dev, st, half, mods);
    case Kind::kLatency: return launch_variant<Lat>(p, dev, st, half, mods);
    default: return launch_variant<Spl>(p, dev, st, half, mods);
  }
}

// Per kernel width (fa_kern_w<W>.cu).
fa_status launch_w16(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w32(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w48(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w64(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w80(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w96(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w128(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);
fa_status launch_w256(Kind, FwdParams &, int dev, cudaStream_t, bool half, bool mods);

}  // namespace fab
