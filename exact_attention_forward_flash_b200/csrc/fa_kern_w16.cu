// fa_kern_w16.cu -- the forward kernels of width 16 (head dim 16).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd16 = FwdCfg<16, 128, 3, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Two16 = FwdCfg<16, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat16 = FwdCfg<16, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl16 = FwdCfg<16, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w16(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two16>(p, dev, st, half, mods);
  return launch_kind<Fwd16, Lat16, Spl16>(k, p, dev, st, half, mods);
}

}  // namespace fab
