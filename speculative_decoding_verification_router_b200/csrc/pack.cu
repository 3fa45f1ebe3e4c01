// Tile-contiguous weight layout for the expert GEMMs.
//
// A weight matrix W[e][r][c] (r rows, c columns = the contraction dim) is
// stored as P[e][r/128][c/64][128][64]: every 128-row x 64-column tile that
// one TMA box loads is one contiguous 16 KB block, so each load streams
// whole DRAM pages instead of 128-byte pieces of many long rows.  The values
// are unchanged; only their order is.
#include "ms_common.cuh"

namespace ms {

__global__ void __launch_bounds__(256) pack_weights_kernel(const uint4* __restrict__ w, int E, int R, int C,
                                                           uint4* __restrict__ out) {
    grid_dep_wait();
    grid_dep_launch();
    // one uint4 = 8 bf16; a tile row of 64 columns = 8 uint4
    const long c8 = C / 8;
    const long total = static_cast<long>(E) * R * c8;
    const int kt = C / 64;
    for (long v = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x; v < total;
         v += static_cast<long>(gridDim.x) * blockDim.x) {
        // v enumerates the OUTPUT in order: [e][rb][kb][row][q]
        const int q = static_cast<int>(v % 8);
        long rest = v / 8;
        const int row = static_cast<int>(rest % 128);
        rest /= 128;
        const int kb = static_cast<int>(rest % kt);
        rest /= kt;
        const int rb = static_cast<int>(rest % (R / 128));
        const long e = rest / (R / 128);
        const long src = (e * R + static_cast<long>(rb) * 128 + row) * c8 + static_cast<long>(kb) * 8 + q;
        out[v] = __ldg(w + src);
    }
}

}  // namespace ms

extern "C" ms_status moe_pack_weights(const void* w, int E, int rows, int cols, void* packed, void* stream) {
    if (!w || !packed || E <= 0 || rows <= 0 || cols <= 0) return MS_ERR_INVALID_ARG;
    if (rows % 128 != 0 || cols % 64 != 0) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(w) || !ms::aligned16(packed) || w == packed) return MS_ERR_INVALID_ARG;
    const long total = static_cast<long>(E) * rows * (cols / 8);
    const long want = (total + 255) / 256;
    const int grid = static_cast<int>(want < 16L * ms::num_sms() ? want : 16L * ms::num_sms());
    return ms::launch(ms::K_PACK, ms::pack_weights_kernel, dim3(grid), dim3(256), 0,
                      static_cast<cudaStream_t>(stream), static_cast<const uint4*>(w), E, rows, cols,
                      static_cast<uint4*>(packed));
}
