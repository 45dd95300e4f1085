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
// CTA (192 threads, one per SM, persistent over output tiles):
//   warp 0     TMA producer: an X tile [128 x 64] and a W tile per stage,
//              128-byte swizzle (K-major operands).
//   warp 1     TMEM owner; one elected lane issues the UMMAs (K16, four per
//              stage).
//   warps 2-9  epilogue, two warps per TMEM lane quarter (warp % 4), each
//              taking half of a tile's columns for its 32 rows, one output
//              row per thread: bias, rotation from a per-CTA (cos, sin)
//              table, bf16; each warp stages its 32 x 32 chunk in shared
//              memory and one lane writes it with a TMA store (whole
//              64-byte row segments instead of 16-byte pieces of 32 rows).
//              Two warps per sub-partition let one compute while the
//              other waits for its TMEM load.
// Two forms:
//   single CTA   tiles of 128 x BN (BN = 256 when C is a multiple of 256,
//                else 128), UMMA M128 x N = BN, four 48 KB stages.
//   CTA pair     (cluster of two SMs, C a multiple of 256) tiles of
//                256 x 256: each CTA stages its own 128 rows of X and half
//                (128 rows) of the W tile in five 32 KB stages, and the
//                epilogue warps stage their output chunks in two buffers
//                each; the pair's leader issues
//                cta_group::2 UMMAs (M256 x N256) that read both CTAs'
//                shared memory and leave rows 0-127 of the accumulator in
//                the leader's TMEM and rows 128-255 in the peer's.  Per
//                SM, each stage moves 32 KB for the same tensor work a
//                48 KB single-CTA stage feeds, and the L2 -> SM traffic
//                drops by a third.  Both CTAs' copies
//                complete on the leader's full barrier (the leader expects
//                both byte counts); the leader's commits arrive on both
//                CTAs' barriers (one multicast commit); both epilogues
//                release an accumulator on the leader's barrier.
// TMEM holds two accumulators of BN fp32 columns, so the epilogue of one
// tile overlaps the UMMAs of the next.  Tiles run row-block-major: the
// 3C / BN tiles of one row block of X are neighbours, so X is read from
// DRAM about once and W (6 MB at C = 1024) stays in L2.
#pragma once
#include "attn_kernel.cuh"

namespace vggt {

constexpr int kGemmBM = 128;  // X rows one CTA stages (one TMEM lane per row)
constexpr int kGemmBK = 64;
#ifndef VGGT_QKV_EPI_WARPS
#define VGGT_QKV_EPI_WARPS 8
#endif
constexpr int kGemmEpiWarps = VGGT_QKV_EPI_WARPS;  // 4 or 8: one or two per TMEM lane quarter
constexpr int kGemmThreads = 64 + 32 * kGemmEpiWarps;
static_assert(kGemmEpiWarps == 4 || kGemmEpiWarps == 8, "one or two epilogue warps per lane quarter");
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

// Tile geometry of the two forms (BN = output columns of a tile).
template <int BN, bool kPair>
struct QkvCfg {
    static constexpr int kStages = kPair ? 5 : 4;
    static constexpr int kOutBufs = kPair ? 2 : 1;  // output staging buffers per epilogue warp
    static constexpr int kRowsB = kPair ? BN / 2 : BN;            // W rows one CTA stages
    static constexpr int kTileM = kPair ? 2 * kGemmBM : kGemmBM;  // output rows of a tile
    static constexpr uint32_t kCtaBytes = (kGemmBM + kRowsB) * kGemmBK * 2;  // one CTA's stage
};

template <int BN, bool kPair>
struct __align__(1024) QkvSmem {
    using Cfg = QkvCfg<BN, kPair>;
    uint8_t a[Cfg::kStages][kGemmBM * kGemmBK * 2];
    uint8_t b[Cfg::kStages][Cfg::kRowsB * kGemmBK * 2];
    uint8_t out[kGemmEpiWarps][Cfg::kOutBufs][32 * 32 * 2];  // one warp's 32 x 32 bf16 chunk, 64-byte swizzle
    float2 rope[kRopeMaxPos][kRopePairs];  // (cos, sin) of pos * base^(-i/16)
    uint64_t full[Cfg::kStages], empty[Cfg::kStages];
    uint64_t acc_full[2], acc_empty[2];
    uint64_t drain;
    uint32_t tmem_base;
    WaitCtl ctl;
};

template <int BN, bool kPair>
constexpr size_t qkv_smem_bytes()
{
    return sizeof(QkvSmem<BN, kPair>) + 1024;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// 2D tiled TMA store of a shared-memory box at (c0, c1); bulk-group completion.
__device__ __forceinline__ void tma_store_2d(const void *map, uint32_t src, int c0, int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(src), "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit()
{
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// The shared-memory sources of this thread's committed stores have been read.
__device__ __forceinline__ void bulk_wait_read_all()
{
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// This thread's committed stores have completed.
__device__ __forceinline__ void bulk_wait_all()
{
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// ------------------------------------------------- CTA-pair (cta_group::2)

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_count_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Every thread of both CTAs; orders the shared-memory writes before it
// (barrier initialisation, TMEM address) for the other CTA.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive once on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// 2D tiled load into this CTA's shared memory that completes on an
// mbarrier of either CTA of the pair (shared::cluster address); no
// multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void *map, uint32_t cluster_bar, int c0,
                                                 int c1)
{
    asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(cluster_bar), "r"(c0), "r"(c1)
                 : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D (M256, split across the pair's TMEM) (+)= A (128 rows in each CTA) *
// B (half of N in each CTA); issued by the leader CTA only.
__device__ __forceinline__ void umma_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrive once on the mbarrier at offset `bar` in both CTAs of the pair when
// every UMMA the leader issued so far has completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::
                     "r"(bar),
                 "h"(static_cast<uint16_t>(3))
                 : "memory");
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
    unsigned long long wait_limit_ns;
};

// Store maps of the C-wide output blocks (Q, K, V; only the first for the
// output projection): [S rows][C columns] bf16, 32 x 32 boxes, 64-byte
// swizzle.
struct QkvOutMaps {
    CUtensorMap m[3];
};

// Where a CTA sits in the launch: tiles pair, pair + n_pairs, ... are its;
// rank is its place in the CTA pair (0 = leader; always 0 single-CTA).
struct QkvSeat {
    uint32_t rank;
    int pair, n_pairs;
};

template <int BN, bool kPair>
__device__ __forceinline__ void qkv_producer(QkvSmem<BN, kPair> &sm, const CUtensorMap *tmX, const CUtensorMap *tmW,
                                             const QkvParams &p, const QkvSeat seat)
{
    using Cfg = QkvCfg<BN, kPair>;
    volatile WaitCtl *ab = &sm.ctl;
    const bool leader = elect_one();
    uint32_t u = 0;  // stages issued
    for (int tile = seat.pair; tile < p.n_tiles; tile += seat.n_pairs) {
        const int m0 = (tile / p.n_tiles_n) * Cfg::kTileM + static_cast<int>(seat.rank) * kGemmBM;
        const int n0 = (tile % p.n_tiles_n) * BN + static_cast<int>(seat.rank) * Cfg::kRowsB;
        for (int kc = 0; kc < p.k_chunks; ++kc) {
            const uint32_t st = u % Cfg::kStages, ph = ((u / Cfg::kStages) & 1) ^ 1;
            if (!wait_bar_warp(smem_u32(&sm.empty[st]), ph, ab, kSiteGemmEmpty))
                goto out;
            if (leader) {
                const uint32_t full = smem_u32(&sm.full[st]);
                if constexpr (kPair) {
                    // Both CTAs' copies complete on the leader's barrier,
                    // which expects both byte counts.
                    if (seat.rank == 0)
                        mbar_arrive_expect_tx(full, 2 * Cfg::kCtaBytes);
                    const uint32_t bar = mapa_shared(full, 0);
                    tma_load_2d_pair(smem_u32(sm.a[st]), tmX, bar, kc * kGemmBK, m0);
                    tma_load_2d_pair(smem_u32(sm.b[st]), tmW, bar, kc * kGemmBK, n0);
                } else {
                    mbar_arrive_expect_tx(full, Cfg::kCtaBytes);
                    tma_load_2d(smem_u32(sm.a[st]), tmX, full, kc * kGemmBK, m0);
                    tma_load_2d(smem_u32(sm.b[st]), tmW, full, kc * kGemmBK, n0);
                }
            }
            ++u;
        }
    }
out:
    // Every copy this warp started must land before the CTA may exit.  The
    // pair's follower cannot watch its copies (they complete on the
    // leader's barrier): on a clean run the leader's last UMMA consumed
    // them all before the pair's final barrier; after an aborted wait it
    // gives them a bounded grace period instead.
    if (leader) {
        if (!kPair || seat.rank == 0) {
            for (uint32_t x = (u > Cfg::kStages ? u - Cfg::kStages : 0); x < u; ++x)
                wait_drain(smem_u32(&sm.full[x % Cfg::kStages]), (x / Cfg::kStages) & 1);
        } else if (ab->abort) {
            const uint64_t t0 = globaltimer_ns();
            while (globaltimer_ns() - t0 < 200000ull)
                __nanosleep(1000);
        }
    }
    __syncwarp();
}

// One thread (the pair's leader CTA only, in the pair form).  Accumulator b
// of tile tl is free once the epilogue(s) have read its previous use
// (acc_empty); a stage is released after its four UMMAs.
template <int BN, bool kPair>
__device__ __forceinline__ void qkv_mma(QkvSmem<BN, kPair> &sm, uint32_t tmem, const QkvParams &p,
                                        volatile WaitCtl *ab, const QkvSeat seat)
{
    using Cfg = QkvCfg<BN, kPair>;
    constexpr uint32_t kIdesc = idesc_bf16_f32(Cfg::kTileM, BN, false);
    constexpr uint64_t kStepA = (kGemmBM * kGemmBK * 2) >> 4;
    constexpr uint64_t kStepB = (Cfg::kRowsB * kGemmBK * 2) >> 4;
    const uint64_t da0 = sdesc_sw128(smem_u32(sm.a[0]), 16, 1024);
    const uint64_t db0 = sdesc_sw128(smem_u32(sm.b[0]), 16, 1024);
    uint32_t u = 0, tl = 0;
    for (int tile = seat.pair; tile < p.n_tiles; tile += seat.n_pairs, ++tl) {
        const uint32_t b = tl & 1;
        if (!wait_bar(smem_u32(&sm.acc_empty[b]), ((tl >> 1) & 1) ^ 1, ab, kSiteAccEmpty))
            return;
        tc_fence_after();
        const uint32_t d = tmem + b * BN;
        for (int kc = 0; kc < p.k_chunks; ++kc, ++u) {
            const uint32_t st = u % Cfg::kStages, ph = (u / Cfg::kStages) & 1;
            if (!wait_bar(smem_u32(&sm.full[st]), ph, ab, kSiteGemmFull))
                return;
            tc_fence_after();
            const uint64_t a = da0 + st * kStepA, bb = db0 + st * kStepB;
#pragma unroll
            for (int kk = 0; kk < kGemmBK / 16; ++kk) {
                if constexpr (kPair)
                    umma_ss_pair(d, a + 2 * kk, bb + 2 * kk, kIdesc, (kc > 0 || kk > 0) ? 1u : 0u);
                else
                    umma_ss(d, a + 2 * kk, bb + 2 * kk, kIdesc, (kc > 0 || kk > 0) ? 1u : 0u);
            }
            if constexpr (kPair)
                umma_commit_pair(smem_u32(&sm.empty[st]));
            else
                umma_commit(smem_u32(&sm.empty[st]));
        }
        if constexpr (kPair)
            umma_commit_pair(smem_u32(&sm.acc_full[b]));
        else
            umma_commit(smem_u32(&sm.acc_full[b]));
    }
}

template <int BN, bool kPair>
__device__ __forceinline__ void qkv_epilogue(QkvSmem<BN, kPair> &sm, uint32_t tmem, const QkvParams &p,
                                             const QkvOutMaps &om, const QkvSeat seat)
{
    using Cfg = QkvCfg<BN, kPair>;
    volatile WaitCtl *ab = &sm.ctl;
    const int lane = threadIdx.x & 31;
    const int quarter = (threadIdx.x >> 5) & 3;  // TMEM lane quarter of this warp
    constexpr int kParts = kGemmEpiWarps / 4;    // warps sharing a lane quarter
    constexpr int kChunks = BN / 32 / kParts;    // 32-column chunks per warp and tile
    const int ew = (static_cast<int>(threadIdx.x) >> 5) - 2;  // epilogue warp
    const int part = ew / 4;
    const uint32_t out_buf0 = smem_u32(sm.out[ew][0]);
    uint32_t chunk_no = 0;
    const int row = static_cast<int>(seat.rank) * kGemmBM + quarter * 32 + lane;  // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const int C = p.C;
    const bool bias4 = p.bias && (reinterpret_cast<uintptr_t>(p.bias) & 15u) == 0;
    // The pair's accumulators are released on the leader's barriers.
    const uint32_t acc_empty0 = kPair ? mapa_shared(smem_u32(&sm.acc_empty[0]), 0) : smem_u32(&sm.acc_empty[0]);
    const uint32_t acc_empty_step = static_cast<uint32_t>(sizeof(uint64_t));

    // (cos, sin) of pos * base^(-i/16) for every grid position and pair.
    for (int idx = static_cast<int>(threadIdx.x) - 64; idx < kRopeMaxPos * kRopePairs; idx += 32 * kGemmEpiWarps) {
        const int pos = idx / kRopePairs, i = idx - pos * kRopePairs;
        const float theta = exp2f(-static_cast<float>(i) / kRopePairs * p.log2_base);
        float sn, cs;
        sincosf(static_cast<float>(pos) * theta, &sn, &cs);
        sm.rope[pos][i] = make_float2(cs, sn);
    }
    // Every epilogue warp reaches this barrier.
    asm volatile("bar.sync 1, %0;" ::"n"(32 * kGemmEpiWarps) : "memory");

    uint32_t tl = 0;
    for (int tile = seat.pair; tile < p.n_tiles; tile += seat.n_pairs, ++tl) {
        const uint32_t b = tl & 1;
        const int m = (tile / p.n_tiles_n) * Cfg::kTileM + row;
        const int m_warp = m - lane;  // first of this warp's 32 rows
        const int n0 = (tile % p.n_tiles_n) * BN;
        if (!wait_bar_warp(smem_u32(&sm.acc_full[b]), (tl >> 1) & 1, ab, kSiteAccFull))
            break;
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
        for (int j = part * kChunks; j < (part + 1) * kChunks; ++j) {
            uint32_t r[32];
            tmem_ld32(tmem + b * BN + 32 * j + lane_off, r);
            tmem_ld_wait();
            reg_fence(r);
            const int n = n0 + 32 * j;  // global output column of r[0]
            float x[32];
            if (bias4) {
                const float4 *b4 = reinterpret_cast<const float4 *>(p.bias + n);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float4 t = __ldg(b4 + e);
                    x[4 * e] = __uint_as_float(r[4 * e]) + t.x;
                    x[4 * e + 1] = __uint_as_float(r[4 * e + 1]) + t.y;
                    x[4 * e + 2] = __uint_as_float(r[4 * e + 2]) + t.z;
                    x[4 * e + 3] = __uint_as_float(r[4 * e + 3]) + t.w;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    x[e] = __uint_as_float(r[e]) + (p.bias ? __ldg(p.bias + n + e) : 0.f);
            }
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
            // Stage the warp's 32 x 32 chunk (row = lane, 64 B each) in the
            // 64-byte-swizzled layout the store map reads: 16-byte unit u of
            // row r sits at unit u ^ ((r >> 1) & 3), so the 8 rows of one
            // store wavefront hit distinct banks.  The previous chunk's
            // store must have read the buffer first.
            const uint32_t out_buf = out_buf0 + (Cfg::kOutBufs == 2 ? (chunk_no & 1) * 2048u : 0u);
            ++chunk_no;
            if (lane == 0) {
                if constexpr (Cfg::kOutBufs == 2)
                    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                else
                    bulk_wait_read_all();
            }
            __syncwarp();
            const uint32_t row_addr = out_buf + static_cast<uint32_t>(lane) * 64;
            const uint32_t sw = (static_cast<uint32_t>(lane) >> 1) & 3;
#pragma unroll
            for (int g = 0; g < 4; ++g)
                st_shared_v4(row_addr + ((static_cast<uint32_t>(g) ^ sw) << 4), pack_bf16x2(x[8 * g], x[8 * g + 1]),
                             pack_bf16x2(x[8 * g + 2], x[8 * g + 3]), pack_bf16x2(x[8 * g + 4], x[8 * g + 5]),
                             pack_bf16x2(x[8 * g + 6], x[8 * g + 7]));
            fence_proxy_async_smem();
            __syncwarp();
            // Rows past S are clipped by the store; a box wholly past S is
            // not issued.
            if (lane == 0) {
                if (m_warp < p.S && VGGT_IN_RANGE(m_warp >= 0 && n + 32 <= p.n_out, kCheckQkvRow))
                    tma_store_2d(&om.m[n / C], out_buf, n % C, m_warp);
                bulk_commit();  // one group per chunk, empty when nothing was stored
            }
        }
        // Every load of accumulator b has completed: the issuer may reuse it.
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
            if constexpr (kPair)
                mbar_arrive_cluster(acc_empty0 + b * acc_empty_step);
            else
                mbar_arrive(acc_empty0 + b * acc_empty_step);
        }
    }
    // The staged chunks must be read, and the stores done, before the CTA exits.
    if (lane == 0)
        bulk_wait_all();
    __syncwarp();
}

// One launch shape for both forms: the pair form is launched as clusters of
// two CTAs (cluster dimension 2 along x).
template <int BN, bool kPair>
__global__ void __launch_bounds__(kGemmThreads, 1)
    qkv_rope_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                    const __grid_constant__ QkvOutMaps tmO, const QkvParams p)
{
    using Cfg = QkvCfg<BN, kPair>;
    extern __shared__ uint8_t smem_raw[];
    QkvSmem<BN, kPair> &sm = *reinterpret_cast<QkvSmem<BN, kPair> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    QkvSeat seat;
    if constexpr (kPair) {
        seat.rank = cluster_ctarank();
        seat.pair = static_cast<int>(cluster_id_x());
        seat.n_pairs = static_cast<int>(cluster_count_x());
    } else {
        seat.rank = 0;
        seat.pair = static_cast<int>(blockIdx.x);
        seat.n_pairs = static_cast<int>(gridDim.x);
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < Cfg::kStages; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.acc_full[i]), 1);
            mbar_init(smem_u32(&sm.acc_empty[i]), (kPair ? 2 : 1) * kGemmEpiWarps);  // warps releasing it
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
        for (int i = 0; i < 3 && i * p.C < p.n_out; ++i)
            prefetch_tensormap(&tmO.m[i]);
    }
    if (warp == 1) {
        if constexpr (kPair) {
            tmem_alloc_pair(smem_u32(&sm.tmem_base), 2 * BN);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(&sm.tmem_base), 2 * BN);
            tmem_relinquish();
        }
    }
    tc_fence_before();
    __syncthreads();
    if constexpr (kPair)
        cluster_sync_all();  // the other CTA's barriers are initialised
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        qkv_producer<BN, kPair>(sm, &tmX, &tmW, p, seat);
    } else if (warp == 1) {
        volatile WaitCtl *ab = &sm.ctl;
        if (seat.rank == 0 && elect_one()) {
            qkv_mma<BN, kPair>(sm, tmem, p, ab, seat);
            // Every UMMA issued must complete before TMEM is released (and,
            // in the pair form, before the follower's shared memory goes).
            if constexpr (kPair)
                umma_commit_pair(smem_u32(&sm.drain));
            else
                umma_commit(smem_u32(&sm.drain));
            wait_drain(smem_u32(&sm.drain), 0);
        }
        __syncwarp();
    } else {
        qkv_epilogue<BN, kPair>(sm, tmem, p, tmO, seat);
    }

    tc_fence_before();
    __syncthreads();
    // Neither CTA of a pair leaves while the other may still arrive on its
    // barriers or (leader) read its shared memory.
    if constexpr (kPair)
        cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if constexpr (kPair)
            tmem_dealloc_pair(tmem, 2 * BN);
        else
            tmem_dealloc(tmem, 2 * BN);
    }
}

} // namespace vggt
