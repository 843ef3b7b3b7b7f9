// fa_kern_w64.cu -- the forward kernels of width 64 (head dim 64).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd64 = FwdCfg<64, 64, 3, 1, 5, 0, H, false, M>;
template <bool H, bool M> using Two64 = FwdCfg<64, 128, 2, 1, 3, 0, H, false, M>;
template <bool H, bool M> using Lat64 = FwdCfg<64, 128, 1, 2, 3, 3, H, false, M>;
template <bool H, bool M> using Spl64 = FwdCfg<64, 128, 1, 2, 3, 3, H, true, M>;

fa_status launch_w64(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  if (k == Kind::kTwoTile) return launch_variant<Two64>(p, dev, st, half, mods);
  return launch_kind<Fwd64, Lat64, Spl64>(k, p, dev, st, half, mods);
}

}  // namespace fab
