// fa_kern_w80.cu -- the forward kernels of width 80 (head dims 56, 72 and 80).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd80 = FwdCfg<80, 64, 3, 1, 5, 0, H, false, M>;
template <bool H, bool M> using Two80 = FwdCfg<80, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat80 = FwdCfg<80, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl80 = FwdCfg<80, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w80(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two80>(p, dev, st, half, mods);
  return launch_kind<Fwd80, Lat80, Spl80>(k, p, dev, st, half, mods);
}

}  // namespace fab
