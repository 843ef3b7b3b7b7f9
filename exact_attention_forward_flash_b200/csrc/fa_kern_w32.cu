// fa_kern_w32.cu -- the forward kernels of width 32 (head dims 24 and 32).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd32 = FwdCfg<32, 128, 3, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Two32 = FwdCfg<32, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat32 = FwdCfg<32, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl32 = FwdCfg<32, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w32(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two32>(p, dev, st, half, mods);
  return launch_kind<Fwd32, Lat32, Spl32>(k, p, dev, st, half, mods);
}

}  // namespace fab
