// fa_kern_w256.cu -- the forward kernels of width 256 (head dims 136 .. 256,
// in steps of 8): the CTA-pair kernel (units of 256 rows over two SMs,
// 128-key tiles) for forwards, and the one-tile kernel (64-key tiles,
// separate K and V rings) for split-KV partials.
#include "fa_fwd_pair.cuh"
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd256 = FwdCfg<256, 64, 1, 2, 3, 2, H, false, M>;
template <bool H, bool M> using Spl256 = FwdCfg<256, 64, 1, 2, 2, 2, H, true, M>;

// The pair kernel runs as clusters of two CTAs: one pair per unit, at most
// one pair per two SMs.
template <class C>
fa_status launch_pair(FwdParams &p, int dev, cudaStream_t st) {
  static bool configured[kMaxDev] = {false};
  if (dev >= 0 && dev < kMaxDev && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(fa_fwd_pair_kernel<C>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kSmemBytes);
    if (e != cudaSuccess)
      return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    configured[dev] = true;
  }
  p.compact = (p.m_major && p.B >= 1 && p.B <= C::kMaxSchedB) ? 1 : 0;
  const int pairs = std::max(1, std::min(p.num_units, num_sms(dev) / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(C::kThreads, 1, 1);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, fa_fwd_pair_kernel<C>, p);
  if (e == cudaSuccess) e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "pair kernel launch: %s", cudaGetErrorString(e));
  return FA_OK;
}

template <bool H, bool M> struct PairLaunch {
  static fa_status run(FwdParams &p, int dev, cudaStream_t st) {
    return launch_pair<FwdPairCfg<H, M>>(p, dev, st);
  }
};

fa_status launch_w256(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kPair) {
    if (half) return mods ? PairLaunch<true, true>::run(p, dev, st) : PairLaunch<true, false>::run(p, dev, st);
    return mods ? PairLaunch<false, true>::run(p, dev, st) : PairLaunch<false, false>::run(p, dev, st);
  }
  return launch_kind<Fwd256, Fwd256, Spl256>(k, p, dev, st, half, mods);
}

}  // namespace fab
