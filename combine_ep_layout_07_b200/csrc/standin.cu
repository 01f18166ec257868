// Deterministic stand-in for the expert FFN: expert e scales each of its
// rows by 1 + e/E in IEEE fp32 and rounds to bf16 (nearest, ties to even).
// It takes the place of the grouped GEMM that consumes the expanded rows
// (DeepEP issue #48, answer on DeepGEMM needing one row per expert), the way
// the DeepEP issue #760 reproduction fills the expert output with a value
// derived from the routing instead of running a GEMM.
#include <cuda_bf16.h>

#include "epx_internal.cuh"

namespace epx {
namespace {

// expert owning row p: the largest e with off_e[e] <= p (empty experts share
// their offset with the next one, so "largest" skips them)
__device__ __forceinline__ int expert_of_row(const int32_t *off_e, int E, int p)
{
    int lo = 0, hi = E - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off_e[mid] <= p)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(128) standin_kernel(StandinParams p)
{
    if (p.early_pdl) pdl_launch_dependents();
    pdl_wait_previous();
    const int64_t n_route = p.totals[0];
    const int64_t rows = n_route < p.rows ? n_route : p.rows;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const int e = expert_of_row(p.off_e, p.E, (int)row);
        const float scale = __fadd_rn(1.0f, __fdiv_rn((float)e, (float)p.E));
        const int v0 = blockIdx.x * p.vpc;
        const int v1 = min(p.V, v0 + p.vpc);
        for (int v = v0 + threadIdx.x; v < v1; v += blockDim.x) {
            const uint4 q = ld_v4(p.ex + (size_t)row * p.V + v);
            const uint32_t u[4] = {q.x, q.y, q.z, q.w};
            uint32_t o[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float lo = __fmul_rn(__uint_as_float(u[i] << 16), scale);
                const float hi = __fmul_rn(__uint_as_float(u[i] & 0xffff0000u), scale);
                __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
                o[i] = *reinterpret_cast<uint32_t *>(&b);
            }
            st_v4(p.y + (size_t)row * p.V + v, make_uint4(o[0], o[1], o[2], o[3]));
        }
    }
    pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_standin(const StandinParams &p0, cudaStream_t s)
{
    StandinParams p = p0;
    if (p.rows <= 0) return cudaSuccess;
    const int chunks = (p.V + 255) / 256;
    p.vpc = (p.V + chunks - 1) / chunks;
    const int64_t gy = p.rows < 65535 ? p.rows : 65535;
    p.early_pdl = early_trigger((long long)chunks * gy);
    return launch_pdl(standin_kernel, dim3(chunks, (unsigned)gy), dim3(128), 0, s, p);
}

}  // namespace epx
