// sga_kernels.cuh -- the integer and bandwidth-bound parts of AVGGT's
// Subsampled Global Attention ("AVGGT: Rethinking Global Attention for
// Accelerating VGGT", technical summary section 3, step two):
//  * sga_index_kernel: kept-token list and per-token multiplicity
//    M_t = |D| - [t in D] from the window-centre rule (one representative
//    patch per s_h x s_w window; all special tokens kept);
//  * sga_gather_meanfill_kernel: one pass over every K/V row that (a) copies
//    the kept rows (special tokens and window centres) into contiguous
//    buffers for the attention kernel's TMA, (b) sums every patch
//    key/value ("total") and (c) sums the kept patch keys/values ("kept"),
//    in fp32, per block;
//  * sga_finalize_kernel: kbar = (total - kept) / |D| (likewise vbar), a
//    fixed-order reduction over the per-block partial sums.
#pragma once
#include <cstdint>

#include "device_error.cuh"
#include "ptx.cuh"

namespace vggt {

// At most this many blocks (partial-sum slots in the workspace); a launch
// uses min(kMeanfillBlocks, 4 per SM).
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
            if (VGGT_IN_RANGE(n * L + p < S, kCheckIndexToken))
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

// Where in-frame position p goes: its slot among the frame's kept tokens
// (special tokens first, then the kept patches row-major), with
// kSlotSpecial set for a special token (kept, not in the patch sums), or -1
// for a dropped patch.
constexpr int kSlotSpecial = 1 << 30;
__device__ __forceinline__ int frame_slot(int p, int n_special, int h, int w, int s_h, int s_w, int kept_w)
{
    if (p < n_special)
        return p | kSlotSpecial;
    const int g = p - n_special, row = g / w, col = g - row * w;
    if (row != window_centre(row, s_h, h) || col != window_centre(col, s_w, w))
        return -1;
    return n_special + (row / s_h) * kept_w + col / s_w;
}

// Frames up to this many tokens get a per-block table of frame_slot in
// shared memory (4 bytes per position); longer frames compute it per row.
constexpr int kSlotTableMax = 4096;

// Row = one token's H*64 bf16 values = vpr 16-byte vectors per tensor.
// Thread `tid` owns vector (tid % vpr) of tensor (tid / vpr) & 1 (K, then V)
// of rows (tid / (2 vpr)) + k * rps, rps = blockDim / (2 vpr), so its fp32
// accumulators always hold the same 8 columns of one tensor.
//
// One pass over every token row of K and V, the block's rows a contiguous
// chunk of [0, S):
//  * a special token's row is copied to its place in the gathered buffers
//    kc / vc (special tokens are kept but are not part of the patch sums);
//  * a patch row is added to the "total" sums; when the patch is the centre
//    of its window (the kept rule of sga_index_kernel) it is also added to
//    the "kept" sums and copied to its place in kc / vc.
// The place of kept token (frame n, in-frame kept slot a) is n * kpf + a,
// kpf = n_special + kept_h * kept_w, slots in token order: the order of the
// index list.  A thread follows its rows' (frame, position) incrementally
// and looks the slot up in the block's table, so the per-row work is a few
// integer operations per 16 bytes moved.  partial[b][0][col] = block b's K
// total minus K kept, partial[b][1][col] = the same for V.
// kMaxThreads = 256 (4 blocks per SM) serves up to 16 heads; 1024 (one
// block per SM) serves up to 64.
template <int kMaxThreads>
__global__ void __launch_bounds__(kMaxThreads, 1024 / kMaxThreads) sga_gather_meanfill_kernel(
    const uint4 *__restrict__ k, const uint4 *__restrict__ v, int S, int L, int n_special, int h, int w,
    int s_h, int s_w, int n_kept, int vpr, float *__restrict__ partial, uint4 *__restrict__ kc,
    uint4 *__restrict__ vc)
{
    extern __shared__ float red[];  // [rps][2][vpr * 8], then the slot table [L] when L <= kSlotTableMax
    int *slot_tab = reinterpret_cast<int *>(red + blockDim.x * 8);
    const bool table = L <= kSlotTableMax;
    const int tid = threadIdx.x;
    const int rps = blockDim.x / (2 * vpr);
    const int vec = tid % vpr, which = (tid / vpr) & 1, sub = tid / (2 * vpr);
    const uint4 *__restrict__ src = which ? v : k;
    uint4 *__restrict__ out = which ? vc : kc;
    const int per = (S + gridDim.x - 1) / gridDim.x;
    const int r0 = min(S, static_cast<int>(blockIdx.x) * per), r1 = min(S, r0 + per);
    const int kept_w = (w + s_w - 1) / s_w;
    const int kpf = n_special + ((h + s_h - 1) / s_h) * kept_w;
    if (table)
        for (int q = tid; q < L; q += blockDim.x)
            slot_tab[q] = frame_slot(q, n_special, h, w, s_h, s_w, kept_w);
    __syncthreads();

    float tot[8] = {0, 0, 0, 0, 0, 0, 0, 0}, kept[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (sub < rps && r0 + sub < r1) {
        // (frame, position) of the thread's next row, advanced by rps per row
        int n = (r0 + sub) / L, pos = (r0 + sub) - n * L;
        for (int r = r0 + sub; r < r1; r += rps * kMeanfillUnroll) {
            uint4 x[kMeanfillUnroll];
            int dst[kMeanfillUnroll];  // place in kc / vc, or -1 (dropped patch)
            bool live[kMeanfillUnroll], patch[kMeanfillUnroll];
#pragma unroll
            for (int u = 0; u < kMeanfillUnroll; ++u) {
                const int t = r + u * rps;
                live[u] = t < r1;
                dst[u] = -1;
                patch[u] = false;
                if (live[u] && VGGT_IN_RANGE(t >= 0 && t < S && pos == t - n * L, kCheckMeanfillRead)) {
                    x[u] = __ldcs(src + static_cast<size_t>(t) * vpr + vec);
                    const int code = table ? slot_tab[pos] : frame_slot(pos, n_special, h, w, s_h, s_w, kept_w);
                    patch[u] = code < 0 || (code & kSlotSpecial) == 0;  // dropped or kept patch
                    if (code >= 0)
                        dst[u] = n * kpf + (code & (kSlotSpecial - 1));
                }
                pos += rps;
                while (pos >= L) {
                    pos -= L;
                    ++n;
                }
            }
#pragma unroll
            for (int u = 0; u < kMeanfillUnroll; ++u) {
                if (!live[u])
                    continue;
                if (dst[u] >= 0 && VGGT_IN_RANGE(dst[u] < n_kept, kCheckMeanfillSlot))
                    out[static_cast<size_t>(dst[u]) * vpr + vec] = x[u];
                if (patch[u]) {
                    acc8(tot, x[u]);
                    if (dst[u] >= 0)
                        acc8(kept, x[u]);
                }
            }
        }
    }
    // Fixed-order reduction over the rps row groups of the block.
    const int cols = vpr * 8;
    if (sub < rps) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            red[(sub * 2 + which) * cols + vec * 8 + e] = tot[e] - kept[e];
    }
    __syncthreads();
    for (int col = tid; col < 2 * cols; col += blockDim.x) {
        const int wh = col / cols, c = col % cols;
        float s = 0.f;
        for (int g = 0; g < rps; ++g)
            s += red[(g * 2 + wh) * cols + c];
        partial[(static_cast<size_t>(blockIdx.x) * 2 + wh) * cols + c] = s;
    }
}

// kbar[c] = (sum over blocks of (total - kept)) / |D|; likewise vbar.  Each
// block owns kFinalizeCols output columns; its 256 threads sum the block
// partials in 16 interleaved groups, then the groups are added in order,
// so the result does not depend on scheduling.
constexpr int kFinalizeCols = 16;
__global__ void __launch_bounds__(256) sga_finalize_kernel(const float *__restrict__ partial, int hd, int n_dropped,
                                                           int blocks, float *__restrict__ kbar,
                                                           float *__restrict__ vbar)
{
    __shared__ float red[256 / kFinalizeCols][kFinalizeCols];
    const int c = threadIdx.x % kFinalizeCols, g = threadIdx.x / kFinalizeCols;
    constexpr int groups = 256 / kFinalizeCols;
    const int col = blockIdx.x * kFinalizeCols + c;  // over the 2 * hd outputs
    const int which = col / hd, cc = col - which * hd;
    float s = 0.f;
    if (col < 2 * hd)
        for (int b = g; b < blocks; b += groups)
            s += partial[(static_cast<size_t>(b) * 2 + which) * hd + cc];
    red[g][c] = s;
    __syncthreads();
    if (g == 0 && col < 2 * hd) {
        float t = 0.f;
        for (int i = 0; i < groups; ++i)
            t += red[i][c];
        (which == 0 ? kbar : vbar)[cc] = t / static_cast<float>(n_dropped);
    }
}

} // namespace vggt
