// fa_kern_w128.cu -- the forward kernels of width 128 (head dims 104 to 128, in steps of 8).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd128 = FwdCfg<128, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat128 = FwdCfg<128, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl128 = FwdCfg<128, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w128(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  return launch_kind<Fwd128, Lat128, Spl128>(k, p, dev, st, half, mods);
}

}  // namespace fab
