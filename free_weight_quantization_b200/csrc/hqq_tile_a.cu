// hqq_tile_a.cu -- the tile engine's 2-, 3- and 4-bit instantiations, and the dispatch over
// every code width (the 1- and 5- to 8-bit instantiations are in hqq_tile_b.cu, compiled in
// parallel).
#include "hqq_tile.cuh"

namespace hqq_impl {

template cudaError_t launch_tile_nb<2>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<3>(const QParams &, int, bool, bool, int64_t, cudaStream_t);
template cudaError_t launch_tile_nb<4>(const QParams &, int, bool, bool, int64_t, cudaStream_t);

cudaError_t launch_tile_engine(const QParams &P, int nbits, int L, bool full, bool direct,
                               int64_t ntiles, cudaStream_t st) {
    switch (nbits) {
    case 1: return launch_tile_nb<1>(P, L, full, false, ntiles, st);
    case 2: return launch_tile_nb<2>(P, L, full, direct, ntiles, st);
    case 3: return launch_tile_nb<3>(P, L, full, false, ntiles, st);
    case 4: return launch_tile_nb<4>(P, L, full, direct, ntiles, st);
    case 5: return launch_tile_nb<5>(P, L, full, false, ntiles, st);
    case 6: return launch_tile_nb<6>(P, L, full, false, ntiles, st);
    case 7: return launch_tile_nb<7>(P, L, full, false, ntiles, st);
    default: return launch_tile_nb<8>(P, L, full, false, ntiles, st);
    }
}

}  // namespace hqq_impl
