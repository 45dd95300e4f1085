// sga_kernels.cuh -- the integer and bandwidth-bound parts of AVGGT's
// Subsampled Global Attention ("AVGGT: Rethinking Global Attention for
// Accelerating VGGT", technical summary section 3, step two):
//  * sga_index_kernel: kept-token list and per-token multiplicity
//    M_t = |D| - [t in D] from the window-centre rule (one representative
//    patch per s_h x s_w window; all special tokens kept);
//  * sga_gather_meanfill_kernel: one pass that (a) gathers the kept K/V rows
//    named by the index list into contiguous buffers for the attention
//    kernel's TMA, (b) sums every patch key/value ("total") and (c) sums the
//    kept patch keys/values ("kept"), in fp32, per block;
//  * sga_finalize_kernel: kbar = (total - kept) / |D| (likewise vbar), a
//    fixed-order reduction over the per-block partial sums.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace vggt {

// At most this many blocks (partial-sum slots in the workspace); a launch
// uses min(kMeanfillBlocks, 4 per SM), split between the two roles in
// proportion to the bytes each role moves.
constexpr int kMeanfillBlocks = 640;
constexpr int kMeanfillUnroll = 4;

// Centre coordinate of the stride-s window that contains x on an axis of
// length n: windows start at multiples of s; a shorter last window keeps its
// own centre (len-1)/2.
__device__ __forceinline__ int window_centre(int x, int s, int n)
{
    const int start = (x / s) * s;
    const int len = min(s, n - start);
    return start + (len - 1) / 2;
}

__global__ void sga_index_kernel(int S, int L, int n_special, int h, int w, int s_h, int s_w, int n_kept,
                                 int n_dropped, int32_t *__restrict__ kept_idx, int32_t *__restrict__ mult)
{
    const int kept_w = (w + s_w - 1) / s_w;
    const int kept_per_frame = n_special + ((h + s_h - 1) / s_h) * kept_w;
    const int total = max(S, n_kept);
    for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
        if (t < S) {
            const int p = t % L;
            int dropped = 0;
            if (p >= n_special) {
                const int r = (p - n_special) / w, c = (p - n_special) % w;
                dropped = (r != window_centre(r, s_h, h) || c != window_centre(c, s_w, w)) ? 1 : 0;
            }
            mult[t] = n_dropped - dropped;
        }
        if (t < n_kept) {
            const int n = t / kept_per_frame, a = t % kept_per_frame;
            int p;
            if (a < n_special) {
                p = a;
            } else {
                const int b = a - n_special;
                const int wr = b / kept_w, wc = b % kept_w;
                const int r = window_centre(wr * s_h, s_h, h), c = window_centre(wc * s_w, s_w, w);
                p = n_special + r * w + c;
            }
            kept_idx[t] = n * L + p;
        }
    }
}

__device__ __forceinline__ void acc8(float (&a)[8], const uint4 x)
{
    a[0] += bf16lo_to_f32(x.x); a[1] += bf16hi_to_f32(x.x);
    a[2] += bf16lo_to_f32(x.y); a[3] += bf16hi_to_f32(x.y);
    a[4] += bf16lo_to_f32(x.z); a[5] += bf16hi_to_f32(x.z);
    a[6] += bf16lo_to_f32(x.w); a[7] += bf16hi_to_f32(x.w);
}

// Row = one token's H*64 bf16 values = vpr 16-byte vectors.  Thread `tid`
// owns vector (tid % vpr) of rows (tid / vpr) + k * rps, rps = blockDim / vpr,
// so its fp32 accumulators always hold the same 8 columns.
// Blocks [0, total_blocks): all patch rows, contiguous chunks.
// Blocks [total_blocks, gridDim.x): kept rows by index list; every kept row
// is copied to kc/vc, kept patch rows are also summed.
// partial[b][0][col] = K sum of block b, partial[b][1][col] = V sum.
__global__ void __launch_bounds__(512, 2) sga_gather_meanfill_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, const int32_t *__restrict__ kept_idx,
    int n_patch_rows, int L, int n_special, int hw, int n_kept, int vpr, int total_blocks,
    float *__restrict__ partial, uint4 *__restrict__ kc, uint4 *__restrict__ vc)
{
    extern __shared__ float red[];  // [rps][2][vpr * 8]
    const int tid = threadIdx.x;
    const int rps = blockDim.x / vpr;
    const int vec = tid % vpr, sub = tid / vpr;
    const bool total_role = static_cast<int>(blockIdx.x) < total_blocks;
    const int nblk = total_role ? total_blocks : static_cast<int>(gridDim.x) - total_blocks;
    const int b = total_role ? static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x) - total_blocks;
    const int nrows = total_role ? n_patch_rows : n_kept;
    const int per = (nrows + nblk - 1) / nblk;
    const int r0 = min(nrows, b * per), r1 = min(nrows, r0 + per);

    float ak[8] = {0, 0, 0, 0, 0, 0, 0, 0}, av[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (sub < rps) {
        for (int r = r0 + sub; r < r1; r += rps * kMeanfillUnroll) {
            uint4 xk[kMeanfillUnroll], xv[kMeanfillUnroll];
            int tok[kMeanfillUnroll];
            bool live[kMeanfillUnroll];
#pragma unroll
            for (int u = 0; u < kMeanfillUnroll; ++u) {
                const int rr = r + u * rps;
                live[u] = rr < r1;
                tok[u] = 0;
                if (live[u]) {
                    if (total_role)
                        tok[u] = (rr / hw) * L + n_special + (rr % hw);
                    else
                        tok[u] = __ldg(kept_idx + rr);
                    const size_t off = static_cast<size_t>(tok[u]) * vpr + vec;
                    xk[u] = __ldcs(k + off);
                    xv[u] = __ldcs(v + off);
                }
            }
#pragma unroll
            for (int u = 0; u < kMeanfillUnroll; ++u) {
                if (!live[u])
                    continue;
                const int rr = r + u * rps;
                if (!total_role) {
                    const size_t dst = static_cast<size_t>(rr) * vpr + vec;
                    kc[dst] = xk[u];
                    vc[dst] = xv[u];
                    if (tok[u] % L < n_special)
                        continue;  // special tokens are kept but not part of the patch sums
                }
                acc8(ak, xk[u]);
                acc8(av, xv[u]);
            }
        }
    }
    // Fixed-order reduction over the rps row groups of the block.
    const int cols = vpr * 8;
    if (sub < rps) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            red[(sub * 2 + 0) * cols + vec * 8 + e] = ak[e];
            red[(sub * 2 + 1) * cols + vec * 8 + e] = av[e];
        }
    }
    __syncthreads();
    for (int col = tid; col < 2 * cols; col += blockDim.x) {
        const int which = col / cols, c = col % cols;
        float s = 0.f;
        for (int g = 0; g < rps; ++g)
            s += red[(g * 2 + which) * cols + c];
        partial[(static_cast<size_t>(blockIdx.x) * 2 + which) * cols + c] = s;
    }
}

// kbar[c] = (sum of total partials - sum of kept partials) / |D|; same for
// vbar.  One thread per output column, partials summed in block order.
__global__ void sga_finalize_kernel(const float *__restrict__ partial, int hd, int n_dropped, int total_blocks,
                                    int blocks, float *__restrict__ kbar, float *__restrict__ vbar)
{
    const int col = blockIdx.x * blockDim.x + threadIdx.x;
    if (col >= 2 * hd)
        return;
    const int which = col / hd, c = col % hd;
    float tot = 0.f, kept = 0.f;
    for (int b = 0; b < total_blocks; ++b)
        tot += partial[(static_cast<size_t>(b) * 2 + which) * hd + c];
    for (int b = total_blocks; b < blocks; ++b)
        kept += partial[(static_cast<size_t>(b) * 2 + which) * hd + c];
    const float mean = (tot - kept) / static_cast<float>(n_dropped);
    (which == 0 ? kbar : vbar)[c] = mean;
}

} // namespace vggt
