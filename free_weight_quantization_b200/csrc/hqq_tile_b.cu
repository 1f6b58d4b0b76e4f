// hqq_tile_b.cu -- the tile engine's 1-bit and 5- to 8-bit instantiations (compiled apart from
// the 2- to 4-bit ones so that the two build in parallel).
#include "hqq_tile.cuh"

namespace hqq_impl {

template cudaError_t launch_tile_nb<1>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<5>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<6>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<7>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<8>(const QParams &, int, bool, bool, int64_t, cudaStream_t);

}  // namespace hqq_impl
