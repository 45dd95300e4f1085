// register_kernels.cuh -- gather / scatter of the special (register and
// camera) tokens for register attention (VGGT-Omega notes, improvement one
// "Register Attention": in some global layers only the 16 registers plus the
// camera token of every frame attend across frames).  The attention itself
// is the global-attention kernel run over the gathered tokens.
#pragma once
#include <cstdint>

#include "device_error.cuh"

namespace vggt {

// Row r of the gathered sequence is special token (r % ns) of frame r / ns,
// i.e. token (r / ns) * L + r % ns.  One 16-byte vector per thread step;
// Q, K and V are gathered together.
__global__ void special_gather_kernel(const uint4 *__restrict__ q, const uint4 *__restrict__ k,
                                      const uint4 *__restrict__ v, uint4 *__restrict__ qc,
                                      uint4 *__restrict__ kc, uint4 *__restrict__ vc, int rows, int ns, int L,
                                      int vpr)
{
    const int64_t total = static_cast<int64_t>(rows) * vpr;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(i / vpr), e = static_cast<int>(i % vpr);
        const int64_t src = (static_cast<int64_t>(r / ns) * L + r % ns) * vpr + e;
        if (!VGGT_IN_RANGE(r % ns < L, kCheckRegisterRow))
            continue;
        qc[i] = __ldg(q + src);
        kc[i] = __ldg(k + src);
        vc[i] = __ldg(v + src);
    }
}

// Writes the gathered outputs back to the special-token rows of O (and lse,
// H floats per token, when requested); every other row is left untouched.
__global__ void special_scatter_kernel(const uint4 *__restrict__ oc, const float *__restrict__ lsec,
                                       uint4 *__restrict__ o, float *__restrict__ lse, int rows, int ns, int L,
                                       int vpr, int H)
{
    const int64_t total = static_cast<int64_t>(rows) * vpr;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int r = static_cast<int>(i / vpr), e = static_cast<int>(i % vpr);
        const int64_t t = static_cast<int64_t>(r / ns) * L + r % ns;
        if (!VGGT_IN_RANGE(r % ns < L, kCheckRegisterRow))
            continue;
        o[t * vpr + e] = oc[i];
        if (lse && e < H)
            lse[t * H + e] = lsec[static_cast<int64_t>(r) * H + e];
    }
}

} // namespace vggt
