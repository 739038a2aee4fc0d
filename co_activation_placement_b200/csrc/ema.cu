// Exponential moving averages of the co-activation counts, and Ochiai on them.
//
// "Cobalt", "Key Observation": the layout planner tracks an EMA of the tokens
// selecting both experts i and j (and of each expert's load, the diagonal) and
// measures co-activation with Ochiai on those averages.  Per cell, in fp64:
//     ema_out = alpha * C + (1 - alpha) * ema_in     (ema_out = C for the first batch)
//     ochiai  = ema_ij / sqrt(ema_ii * ema_jj), rounded once to fp32 (0 if the product is 0),
// each operation IEEE-rounded (__dmul_rn, __dadd_rn, __dsqrt_rn, __ddiv_rn), no
// fused multiply-add, so the result is fixed by the formula.  Out of place:
// every block recomputes the diagonal it needs from the inputs, so one launch
// has no ordering between blocks.  An HBM stream: 4 + 8 bytes read, 8 + 4
// written per cell.
#include "common.cuh"

namespace moe {
namespace {

constexpr int kEmaThreads = 256;

__device__ __forceinline__ double ema_cell(uint32_t c, const double *__restrict__ ema_in, size_t idx, double alpha,
                                           double beta)
{
    const double x = (double)c;
    if (!ema_in) return x;
    return __dadd_rn(__dmul_rn(alpha, x), __dmul_rn(beta, __ldg(ema_in + idx)));
}

__global__ void __launch_bounds__(kEmaThreads)
coact_ema_kernel(const uint32_t *__restrict__ coact, int E, double alpha, const double *__restrict__ ema_in,
                 double *__restrict__ ema_out, float *__restrict__ ochiai)
{
    extern __shared__ double ediag[];
    const int l = blockIdx.y;
    const size_t EE = (size_t)E * E;
    const double beta = 1.0 - alpha;
    const uint32_t *c_l = coact + (size_t)l * EE;
    const double *in_l = ema_in ? ema_in + (size_t)l * EE : nullptr;
    if (ochiai) {
        for (int e = threadIdx.x; e < E; e += kEmaThreads)
            ediag[e] = ema_cell(__ldg(c_l + (size_t)e * E + e), in_l, (size_t)e * E + e, alpha, beta);
        __syncthreads();
    }
    const size_t c = (size_t)blockIdx.x * kEmaThreads + threadIdx.x;
    if (c >= EE) return;
    const double v = ema_cell(__ldg(c_l + c), in_l, c, alpha, beta);
    ema_out[(size_t)l * EE + c] = v;
    if (ochiai) {
        const int i = (int)(c / E), j = (int)(c % E);
        const double den = __dmul_rn(ediag[i], ediag[j]);
        ochiai[(size_t)l * EE + c] = den > 0.0 ? __double2float_rn(__ddiv_rn(v, __dsqrt_rn(den))) : 0.0f;
    }
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_coact_ema(const uint32_t *coact, int L, int E, double alpha, const double *ema_in,
                                    double *ema_out, float *ochiai, cudaStream_t stream)
{
    if (L < 1 || E < 1 || E > 4096 || !coact || !ema_out) return MOE_ERR_ARG;
    if (!(alpha >= 0.0 && alpha <= 1.0)) return MOE_ERR_ARG;
    if (ema_in && ema_in == ema_out) return MOE_ERR_ARG;
    const size_t EE = (size_t)E * E;
    dim3 grid((unsigned)((EE + kEmaThreads - 1) / kEmaThreads), (unsigned)L);
    const size_t smem = ochiai ? sizeof(double) * E : 0;
    if (allow_smem(coact_ema_kernel, smem) != cudaSuccess) return MOE_ERR_CUDA;
    coact_ema_kernel<<<grid, kEmaThreads, smem, stream>>>(coact, E, alpha, ema_in, ema_out, ochiai);
    moe_status st = launch_status();
    if (st == MOE_OK) note_launches(1);
    return st;
}
