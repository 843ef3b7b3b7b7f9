// fa_kern_w48.cu -- the forward kernels of width 48 (head dims 40 and 48).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd48 = FwdCfg<48, 64, 3, 1, 5, 0, H, false, M>;
template <bool H, bool M> using Two48 = FwdCfg<48, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat48 = FwdCfg<48, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl48 = FwdCfg<48, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w48(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two48>(p, dev, st, half, mods);
  return launch_kind<Fwd48, Lat48, Spl48>(k, p, dev, st, half, mods);
}

}  // namespace fab
