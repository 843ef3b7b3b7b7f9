// fa_kern_w256.cu -- the forward kernels of width 256 (head dims 136 .. 256,
// in steps of 8): one Q tile per CTA and 64-key tiles, with separate K and V
// rings; no separate latency shape (every call takes the one-tile kernel).
#include "fa_launch.cuh"

namespace fab {

template <bool H, bool M> using Fwd256 = FwdCfg<256, 64, 1, 2, 3, 2, H, false, M>;
template <bool H, bool M> using Spl256 = FwdCfg<256, 64, 1, 2, 2, 2, H, true, M>;

fa_status launch_w256(Kind k, FwdParams &p, int dev, cudaStream_t st, bool half, bool mods) {
  return launch_kind<Fwd256, Fwd256, Spl256>(k, p, dev, st, half, mods);
}

}  // namespace fab
