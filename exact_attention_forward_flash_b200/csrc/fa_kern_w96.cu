// fa_kern_w96.cu -- the forward kernels of width 96 (head dims 88 and 96).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd96 = FwdCfg<96, 64, 3, 1, 5, 0, H, false, M>;
template <bool H, bool M> using Two96 = FwdCfg<96, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat96 = FwdCfg<96, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl96 = FwdCfg<96, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w96(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two96>(p, dev, st, half, mods);
  return launch_kind<Fwd96, Lat96, Spl96>(k, p, dev, st, half, mods);
}

}  // namespace fab
