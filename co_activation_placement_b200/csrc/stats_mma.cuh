// Tensor-core path of the co-activation statistics (stats_mma.cu), used by
// moe_coact_stats when the expert count suits the tcgen05 shapes.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_coact.h"

namespace moe {

struct MmaGeom {
    int L, T, k, E;
    int rows;    // X tile rows: E rounded up to a multiple of 128
    int mt;      // 128-row M tiles
    int nc;      // C products (L, or 0 when only transitions are wanted)
    int P;       // products: C_0..C_{nc-1}, then M_0..M_{L-2} when wanted
    bool paired; // a block computes C_l and M_l together (both accumulators fit)
    bool quad;   // a block computes C and M of layers 2j and 2j + 1 (E <= 128)
    int J;       // jobs per token slice: (L + 1) / 2 when quad, L when paired, else P
    int S;       // token slices per job
    int cols;    // tensor-memory columns per block (a power of two >= mt*E)
};

// false when the shape is outside the tensor-core path (E % 16 != 0, E < 32,
// E > 256, k > 8, T < 1)
bool make_mma_geom(int L, int T, int k, int E, bool want_c, bool want_t, MmaGeom &g);
size_t mma_smem_bytes(const MmaGeom &g);
size_t mma_partial_words(const MmaGeom &g);
moe_status coact_mma(const int32_t *ids, const MmaGeom &g, uint32_t *part, uint32_t *coact, float *ochiai,
                     uint32_t *trans, int32_t *err, cudaStream_t stream);

}  // namespace moe
