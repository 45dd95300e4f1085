// qkv_kernel.cuh -- fused QKV projection with a 2D rotary position
// embedding on the sm_100a tensor cores: Y = X W^T + b (tcgen05 UMMA, fp32
// accumulators in TMEM, X and W tiles staged by TMA), split into Q, K and V
// in the [S, H, 64] attention layout, Q and K rotated in the epilogue.
//
// What it computes: the projection that produces each attention layer's
// Q, K and V, and a rotary position embedding applied to Q and K before the
// attention ("Feed-forward optimization in Visual Geometry Grounded and
// 3DGS", Cut3R part, section 3.5, position encoding).  The pages give no
// formula; the 2D form used: a patch token at grid (r, c) is rotated by
// position r in the first half of each head's 64 dimensions and by c in the
// second half; within a half, dimensions i and i + 16 form a pair rotated
// by pos * base^(-i/16): a' = a cos - b sin, b' = b cos + a sin; special
// tokens are not rotated.
//
// CTA (192 threads, one per SM, persistent over 128 x BN output tiles,
// BN = 256 when C is a multiple of 256, else 128):
//   warp 0     TMA producer: an X tile [128 x 64] and a W tile [BN x 64]
//              per stage, 128-byte swizzle (K-major operands).
//   warp 1     TMEM owner; one elected lane issues the UMMAs (M128, N = BN,
//              K16, four per stage).
//   warps 2-5  epilogue, one output row per thread (TMEM lane quarter =
//              warp % 4): bias, rotation from a per-CTA (cos, sin) table,
//              bf16, 16-byte stores.
// TMEM holds two accumulators of BN fp32 columns, so the epilogue of one
// tile overlaps the UMMAs of the next.  Tiles run row-block-major: the
// 3C / BN tiles of one 128-row block of X are neighbours, so X is read from
// DRAM about once and W (6 MB at C = 1024) stays in L2.
#pragma once
#include "attn_kernel.cuh"

namespace vggt {

constexpr int kGemmBM = 128;
constexpr int kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 192;
constexpr int kRopeMaxPos = 128;  // grid rows / columns the rotation table covers
constexpr int kRopePairs = 16;    // rotated pairs per 32-dimension half of a head

enum : uint32_t { kSiteGemmFull = 12, kSiteGemmEmpty, kSiteAccFull, kSiteAccEmpty };

// 2D tiled TMA load of box (c0, c1) into shared memory, completing on bar.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void *map, uint32_t bar, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
                 : "memory");
}

template <int BN>
struct __align__(1024) QkvSmem {
    uint8_t a[kGemmStages][kGemmBM * kGemmBK * 2];
    uint8_t b[kGemmStages][BN * kGemmBK * 2];
    float2 rope[kRopeMaxPos][kRopePairs];  // (cos, sin) of pos * base^(-i/16)
    uint64_t full[kGemmStages], empty[kGemmStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    WaitCtl ctl;
};

template <int BN>
constexpr size_t qkv_smem_bytes()
{
    return sizeof(QkvSmem<BN>) + 1024;
}

struct QkvParams {
    int S;          // tokens
    int C;          // H * 64
    int n_out;      // output columns: 3C (QKV projection) or C (output projection)
    int rope_cols;  // leading output columns that are rotated: 2C (Q, K) or 0
    int n_tiles_n;  // n_out / BN
    int n_tiles;    // ceil(S / 128) * n_tiles_n
    int k_chunks;   // C / 64
    int L, n_special, pw;
    float log2_base;
    const float *bias;  // [n_out] or null
    __nv_bfloat16 *q, *k, *v;  // C-wide output blocks 0, 1, 2 (k, v unused when n_out = C)
    unsigned long long wait_limit_ns;
};

template <int BN>
__device__ __forceinline__ void qkv_producer(QkvSmem<BN> &sm, const CUtensorMap *tmX, const CUtensorMap *tmW,
                                             const QkvParams &p)
{
    volatile WaitCtl *ab = &sm.ctl;
    const bool leader = elect_one();
    constexpr uint32_t kBytes = (kGemmBM + BN) * kGemmBK * 2;
    uint32_t u = 0;  // stages issued
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
        const int m0 = (tile / p.n_tiles_n) * kGemmBM;
        const int n0 = (tile % p.n_tiles_n) * BN;
        for (int kc = 0; kc < p.k_chunks; ++kc) {
            const uint32_t st = u % kGemmStages, ph = ((u / kGemmStages) & 1) ^ 1;
            if (!wait_bar_warp(smem_u32(&sm.empty[st]), ph, ab, kSiteGemmEmpty))
                goto out;
            if (leader) {
                mbar_arrive_expect_tx(smem_u32(&sm.full[st]), kBytes);
                tma_load_2d(smem_u32(sm.a[st]), tmX, smem_u32(&sm.full[st]), kc * kGemmBK, m0);
                tma_load_2d(smem_u32(sm.b[st]), tmW, smem_u32(&sm.full[st]), kc * kGemmBK, n0);
            }
            ++u;
        }
    }
out:
    // Every copy this warp started must land before the CTA may exit.
    if (leader)
        for (uint32_t x = (u > kGemmStages ? u - kGemmStages : 0); x < u; ++x)
            wait_drain(smem_u32(&sm.full[x % kGemmStages]), (x / kGemmStages) & 1);
    __syncwarp();
}

// One thread.  Accumulator b of tile tl is free once the epilogue has read
// its previous use (acc_empty); a stage is released after its four UMMAs.
template <int BN>
__device__ __forceinline__ void qkv_mma(QkvSmem<BN> &sm, uint32_t tmem, const QkvParams &p, volatile WaitCtl *ab)
{
    constexpr uint32_t kIdesc = idesc_bf16_f32(kGemmBM, BN, false);
    constexpr uint64_t kStepA = (kGemmBM * kGemmBK * 2) >> 4;
    constexpr uint64_t kStepB = (BN * kGemmBK * 2) >> 4;
    const uint64_t da0 = sdesc_sw128(smem_u32(sm.a[0]), 16, 1024);
    const uint64_t db0 = sdesc_sw128(smem_u32(sm.b[0]), 16, 1024);
    uint32_t u = 0, tl = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++tl) {
        const uint32_t b = tl & 1;
        if (!wait_bar(smem_u32(&sm.acc_empty[b]), ((tl >> 1) & 1) ^ 1, ab, kSiteAccEmpty))
            return;
        tc_fence_after();
        const uint32_t d = tmem + b * BN;
        for (int kc = 0; kc < p.k_chunks; ++kc, ++u) {
            const uint32_t st = u % kGemmStages, ph = (u / kGemmStages) & 1;
            if (!wait_bar(smem_u32(&sm.full[st]), ph, ab, kSiteGemmFull))
                return;
            tc_fence_after();
            const uint64_t a = da0 + st * kStepA, bb = db0 + st * kStepB;
#pragma unroll
            for (int kk = 0; kk < kGemmBK / 16; ++kk)
                umma_ss(d, a + 2 * kk, bb + 2 * kk, kIdesc, (kc > 0 || kk > 0) ? 1u : 0u);
            umma_commit(smem_u32(&sm.empty[st]));
        }
        umma_commit(smem_u32(&sm.acc_full[b]));
    }
}

template <int BN>
__device__ __forceinline__ void qkv_epilogue(QkvSmem<BN> &sm, uint32_t tmem, const QkvParams &p)
{
    volatile WaitCtl *ab = &sm.ctl;
    const int lane = threadIdx.x & 31;
    const int quarter = (threadIdx.x >> 5) & 3;  // TMEM lane quarter of this warp
    const int row = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int C = p.C;

    // (cos, sin) of pos * base^(-i/16) for every grid position and pair.
    for (int idx = static_cast<int>(threadIdx.x) - 64; idx < kRopeMaxPos * kRopePairs; idx += 128) {
        const int pos = idx / kRopePairs, i = idx - pos * kRopePairs;
        const float theta = exp2f(-static_cast<float>(i) / kRopePairs * p.log2_base);
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta, &sn, &cs);
        sm.rope[pos][i] = make_float2(cs, sn);
    }
    // The four epilogue warps (128 threads) all reach this barrier.
    asm volatile("bar.sync 1, 128;" ::: "memory");

    uint32_t tl = 0;
    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x, ++tl) {
        const uint32_t b = tl & 1;
        const int m = (tile / p.n_tiles_n) * kGemmBM + row;
        const int n0 = (tile % p.n_tiles_n) * BN;
        if (!wait_bar_warp(smem_u32(&sm.acc_full[b]), (tl >> 1) & 1, ab, kSiteAccFull))
            return;
        tc_fence_after();
        int pr = 0, pc = 0;  // special tokens (and rows past S) are not rotated
        if (m < p.S) {
            const int pp = m % p.L;
            if (pp >= p.n_special) {
                const int g = pp - p.n_special;
                pr = g / p.pw;
                pc = g - pr * p.pw;
            }
        }
#pragma unroll 1
        for (int j = 0; j < BN / 32; ++j) {
            uint32_t r[32];
            tmem_ld32(tmem + b * BN + 32 * j + lane_off, r);
            tmem_ld_wait();
            reg_fence(r);
            const int n = n0 + 32 * j;  // global output column of r[0]
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; ++e)
                x[e] = __uint_as_float(r[e]) + (p.bias ? __ldg(p.bias + n + e) : 0.f);
            if (n < p.rope_cols) {
                // a 32-column chunk is one half of one head of Q or K
                const int pos = ((n >> 5) & 1) ? pc : pr;
#pragma unroll
                for (int i = 0; i < kRopePairs; ++i) {
                    const float2 t = sm.rope[pos][i];
                    const float a = x[i], c2 = x[i + kRopePairs];
                    x[i] = a * t.x - c2 * t.y;
                    x[i + kRopePairs] = c2 * t.x + a * t.y;
                }
            }
            if (m < p.S && VGGT_IN_RANGE(m >= 0 && n + 32 <= p.n_out, kCheckQkvRow)) {
                __nv_bfloat16 *dst = (n < C ? p.q : (n < 2 * C ? p.k : p.v)) + static_cast<size_t>(m) * C + (n % C);
                uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                for (int g = 0; g < 4; ++g)
                    d4[g] = make_uint4(pack_bf16x2(x[8 * g], x[8 * g + 1]), pack_bf16x2(x[8 * g + 2], x[8 * g + 3]),
                                       pack_bf16x2(x[8 * g + 4], x[8 * g + 5]), pack_bf16x2(x[8 * g + 6], x[8 * g + 7]));
            }
        }
        // Every load of accumulator b has completed: the issuer may reuse it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            mbar_arrive(smem_u32(&sm.acc_empty[b]));
    }
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const QkvParams p)
{
    extern __shared__ uint8_t smem_raw[];
    QkvSmem<BN> &sm = *reinterpret_cast<QkvSmem<BN> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kGemmStages; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.acc_full[i]), 1);
            mbar_init(smem_u32(&sm.acc_empty[i]), 4);
        }
        mbar_init(smem_u32(&sm.drain), 1);
        sm.ctl.abort = 0;
        sm.ctl.limit_ns = p.wait_limit_ns;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmW);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), 2 * BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        qkv_producer<BN>(sm, &tmX, &tmW, p);
    } else if (warp == 1) {
        volatile WaitCtl *ab = &sm.ctl;
        if (elect_one()) {
            qkv_mma<BN>(sm, tmem, p, ab);
            // Every UMMA issued must complete before TMEM is released.
            umma_commit(smem_u32(&sm.drain));
            wait_drain(smem_u32(&sm.drain), 0);
        }
        __syncwarp();
    } else {
        qkv_epilogue<BN>(sm, tmem, p);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, 2 * BN);
    }
}

} // namespace vggt
