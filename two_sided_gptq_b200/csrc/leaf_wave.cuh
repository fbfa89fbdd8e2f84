// leaf_wave.cuh -- launch interface of the continuous strip sweep (leaf
// structure 8, leaf_wave.cu), called by the leaf dispatcher in leaf.cu.
#pragma once

#include "kernels.cuh"

namespace bakron {

// Each CTA of a tile's cluster rounds its 32-row strip in one sweep, 48 steps
// behind the CTA above; tiles I_lo .. I_lo + tiles - 1 of tile diagonal K.
cudaError_t leaf_wave_configure();
cudaError_t launch_leaf_wave(const LeafArgs &p, int K, int I_lo, int tiles, cudaStream_t stream);

}  // namespace bakron
