// attn_kernel.cuh -- flash-style online-softmax attention on the sm_100a
// tensor cores (tcgen05 UMMA, accumulators in TMEM, operands staged by TMA).
//
// One kernel serves the four attention forms of the hot path:
//  * frame attention  -- keys = the query's own frame ("VGGT CVPR25 Best
//    Paper" notes, "Alternating-Attention": frame-wise self-attention);
//  * global attention -- keys = all S tokens (global self-attention);
//  * SGA              -- keys = the gathered kept set, plus the diagonal term
//    and the ln M mean column folded into the same softmax state ("AVGGT:
//    Rethinking Global Attention for Accelerating VGGT", section 3 step two);
//  * register attention -- queries and keys = the special tokens of all
//    frames (VGGT-Omega notes, improvement one "Register Attention"), read in
//    place through 4-D tensor maps: a 128-row tile holds the special tokens
//    of F = floor(128 / n_special) whole frames (n_special * F rows); the
//    rows past them are never loaded, zeroed once at the start and masked.
//
// CTA layout (384 threads, one CTA per SM, persistent over work items):
//   warp 0      TMA producer: Q tiles (double-buffered) and a K/V ring.
//   warp 1      TMEM owner; one elected lane issues every UMMA.
// The producer warp runs its loop converged (warp-uniform operands) and lets
// one elected lane issue the copies.
//   warps 2-3   idle.
//   warps 4-7   softmax warpgroup 0: query rows 0..127 of the item.
//   warps 8-11  softmax warpgroup 1: query rows 128..255.
// Query rows come in 128-row tiles of a unit -- a (frame, head) in frame
// mode, a head otherwise -- and a work item is a pair of consecutive tiles:
// warpgroup 0 takes the first, warpgroup 1 the second.  When both tiles lie
// in one unit they share one K/V stream (one K and one V tile per key step);
// when the pair straddles two units (the last tile of one and the first of
// the next, e.g. at frame ends) each warpgroup streams its own.  Every item
// of a launch has the same number of 128-key tiles.
//
// TMEM (512 columns x 128 lanes x 32 bit): three score buffers SP0 [0,128)
// SP1 [128,256) SP2 [256,384), then O0 [384,448) O1 [448,512).  Lane =
// query row.  S = Q K^T is an SS UMMA (M=128, N=128, K=64 as 4 x K16) into a
// score buffer; the softmax writes P (bf16 pairs) over the first 64 columns
// of the same buffer, and O += P V is a TS UMMA reading P from there and V
// from shared memory (M=128, N=64, K=128 as 8 x K16).
//
// Steps k = 0, 1, 2, ... alternate between the warpgroups (warpgroup k & 1,
// key tile k >> 1) and rotate through the score buffers (buffer k % 3).
// The issuer runs PV(k) as soon as P(k) is written and S(k + 3) as soon as
// PV(k) has completed (its buffer is then free), so scores are computed two
// steps ahead: a warpgroup never waits for a PV before writing P, and its
// next S is normally ready when it finishes the current one.  The softmax
// keeps an offset m in log2 units, set from the row max of an item's first
// key tile; later tiles are exponentiated against m without taking their
// max, and only a tile whose row sum of P exceeds 2^15 takes the exact slow
// path (its max, a rescale of O and l where the max grew by more than 8, P
// again).  Exact for any m, because O and l always share it.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "device_error.cuh"
#include "ptx.cuh"

namespace vggt {

constexpr int kHeadDim = 64;
constexpr int kBlockM = 128;
constexpr int kBlockN = 128;
constexpr int kStages = 4;
constexpr int kAttnThreads = 384;
constexpr uint32_t kTileBytes = kBlockM * kHeadDim * 2;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;    // log2 units: rescale O when the row max grew by more
constexpr float kTileSumLimit = 32768.0f;    // a tile's row sum of P above 2^15 triggers the rescale check
constexpr uint32_t kRegsLaunch = 168;
constexpr uint32_t kRegsControl = 72;
constexpr uint32_t kRegsSoftmax = 216;
static_assert(128 * (kRegsControl + 2 * kRegsSoftmax) <= kAttnThreads * kRegsLaunch,
              "register split exceeds the launch allocation");
// Software 2^x for part of the exponentials (the rest use the MUFU ex2
// unit): Cody-Waite reduction x = j + f, j = round(x), f in [-1/2, 1/2],
// 2^f by the degree-3 polynomial of minimax relative error (Remez exchange;
// coefficients from exp2_poly_fit.py, max relative error 7.5e-5), 2^j added
// to the exponent field.  Of every 16 column pairs of a score row, the first
// kExp2PolyPairs take this path.
#ifndef VGGT_EXP2_POLY_PAIRS
#define VGGT_EXP2_POLY_PAIRS 4
#endif
constexpr int kExp2PolyPairs = VGGT_EXP2_POLY_PAIRS;
constexpr int kScoreBufs = 3;
constexpr uint32_t kTmemO = kScoreBufs * kBlockN;  // first O column
static_assert(kTmemO + 2 * kHeadDim <= kTmemCols, "TMEM layout exceeds 512 columns");
constexpr float kExp2C0 = 0.9999280571937561f;
constexpr float kExp2C1 = 0.6932609677314758f;
constexpr float kExp2C2 = 0.2426111251115799f;
constexpr float kExp2C3 = 0.0551716685295105f;
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr float kExp2MinArg = -125.0f;      // keeps 2^j a normal number
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // default bound of one wait: 4 s
constexpr uint64_t kDrainLimitNs = 200000000ull;  // tail waits before exit: 0.2 s
constexpr uint64_t kPaceLimitNs = 200000ull;      // shortest bound of one pacing wait: 0.2 ms
constexpr int kPaceSlots = 16;                    // pacing counters: one per launch in flight

enum : int { kModeFrame = 0, kModeGlobal = 1, kModeSga = 2, kModeRegister = 3 };

// Wait sites (bits 8..15 of the device error word, see device_error.cuh).
enum : uint32_t {
    kSiteQEmpty = 1, kSiteKEmpty, kSiteVEmpty, kSiteQFull, kSiteKFull, kSiteVFull,
    kSitePReady, kSiteSFull, kSiteODone, kSiteDrain, kSiteOFinal
};

struct AttnParams {
    int mode;
    int S;        // query tokens
    int L;        // tokens per frame
    int H;        // heads
    int n_keys;   // keys per item: L (frame), S (global), n_kept (SGA)
    int n_kt;     // ceil(n_keys / 128)
    int qtiles;   // 128-row query tiles per unit: a (frame, head) in frame mode, a head otherwise
    int n_tiles;  // query tiles of the launch
    int n_items;  // tile pairs, ceil(n_tiles / 2)
    float scale_log2;
    __nv_bfloat16 *o;
    float *lse;
    // SGA only: raw Q/K/V rows for the diagonal term, multiplicities, means.
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    const int32_t *mult;
    const float *kbar;
    const float *vbar;
    int n_dropped;
    int row0;      // SGA on a row block: sequence index of its query row 0 (mult)
    int own_row0;  // SGA: row of k / v holding query row 0's own key and value (the diagonal term)
    // register mode only: frames per tile F, special tokens per frame, frames,
    // and the loaded rows of a tile, n_special * F
    int tile_frames, n_special, n_frames, tile_rows;
    unsigned long long wait_limit_ns;  // bound of one in-kernel wait
    int stall_first_scores;            // test hook: never signal warpgroup 0's first S
    // Item pacing (global attention and SGA): a device counter, zeroed by the
    // host before the launch, of the items whose K/V loads every CTA has
    // issued; nullptr = no pacing.
    unsigned int *pace;
};

// Shared by every bounded wait of a CTA: the abort flag raised by the first
// wait that runs out, and the per-launch bound of one wait.
struct WaitCtl {
    int abort;
    uint32_t pad;
    unsigned long long limit_ns;
};

struct __align__(1024) AttnSmem {
    uint8_t q[2][2][kTileBytes];  // [buffer][warpgroup]
    uint8_t k[kStages][kTileBytes];
    uint8_t v[kStages][kTileBytes];
    uint64_t q_full[2], q_empty[2];
    uint64_t k_full[kStages], k_empty[kStages];
    uint64_t v_full[kStages], v_empty[kStages];
    uint64_t s_full[kScoreBufs], p_ready[2][2], o_done[2], o_final[2];
    uint64_t drain;
    uint32_t tmem_base;
    WaitCtl ctl;
};

constexpr size_t kAttnSmemBytes = sizeof(AttnSmem) + 1024;

struct Work {
    int h, q0, row_end, key0, n_keys;
};

// Query tile t (128 rows): tile t % qtiles of unit t / qtiles.
__device__ __forceinline__ Work tile_work(const AttnParams &p, int t)
{
    Work w;
    const int u = t / p.qtiles, r = t - u * p.qtiles;
    if (p.mode == kModeFrame) {
        const int n = u / p.H;
        w.h = u - n * p.H;
        w.key0 = n * p.L;
        w.q0 = w.key0 + r * kBlockM;
        w.row_end = w.key0 + p.L;
    } else {
        w.h = u;
        w.key0 = 0;
        w.q0 = r * kBlockM;
        w.row_end = p.S;  // register mode: S holds the padded row count, 128 per tile
    }
    w.n_keys = p.n_keys;
    return w;
}

// Whether the two tiles of item `item` lie in different units.
__device__ __forceinline__ bool item_split(const AttnParams &p, int item)
{
    const int t0 = 2 * item;
    return t0 + 1 < p.n_tiles && t0 / p.qtiles != (t0 + 1) / p.qtiles;
}

// The tiles of item `item`: w[0] for warpgroup 0, w[1] for warpgroup 1.
// Past the last tile, warpgroup 1 repeats warpgroup 0's tile (so its loads
// stay in bounds) and owns no row.
struct ItemWork {
    Work w[2];
    bool split;
};

// Warpgroup wg's tile of item `item` alone (the softmax warps need no more).
__device__ __forceinline__ Work wg_work(const AttnParams &p, int item, int wg)
{
    const int t = 2 * item + wg;
    if (t < p.n_tiles)
        return tile_work(p, t);
    Work w = tile_work(p, t - 1);
    w.row_end = w.q0;
    return w;
}

__device__ __forceinline__ ItemWork item_work(const AttnParams &p, int item)
{
    ItemWork iw;
    const int t0 = 2 * item;
    iw.w[0] = tile_work(p, t0);
    if (t0 + 1 < p.n_tiles) {
        iw.w[1] = tile_work(p, t0 + 1);
    } else {
        iw.w[1] = iw.w[0];
        iw.w[1].row_end = iw.w[1].q0;
    }
    iw.split = item_split(p, item);
    return iw;
}

// ------------------------------------------------------------ bounded waits

__device__ __forceinline__ bool wait_slow(uint32_t bar, uint32_t parity, volatile WaitCtl *ctl, uint32_t site)
{
    const uint64_t t0 = globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (ctl->abort)
            return false;
        if (globaltimer_ns() - t0 > ctl->limit_ns) {
            atomicCAS(&g_vggt_error, 0u, kErrTimeout | (site << 8));
            atomicOr(&g_vggt_error, kErrTimeout);
            ctl->abort = 1;
            return false;
        }
    }
}

__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, volatile WaitCtl *ctl, uint32_t site)
{
    if (mbar_try_wait(bar, parity))
        return true;
    return wait_slow(bar, parity, ctl, site);
}

// Warp-uniform wait: lane 0 polls, the verdict is broadcast.
#ifndef VGGT_WARP_POLL
#define VGGT_WARP_POLL 1
#endif
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, volatile WaitCtl *ctl,
                                              uint32_t site)
{
#if VGGT_WARP_POLL
    // Every lane polls: one warp-wide instruction per poll and no shuffle on
    // the way out.  Lanes that see the phase complete in different polls
    // reconverge at the __syncwarp.
    const bool ok = wait_bar(bar, parity, ctl, site);
    __syncwarp();
    return __all_sync(0xffffffffu, ok);
#else
    int ok = 0;
    if ((threadIdx.x & 31) == 0)
        ok = wait_bar(bar, parity, ctl, site) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
#endif
}

// Tail wait used before exit (copies or MMAs in flight); ignores the abort flag.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer_ns() - t0 > kDrainLimitNs) {
            atomicCAS(&g_vggt_error, 0u, kErrTimeout | (kSiteDrain << 8));
            atomicOr(&g_vggt_error, kErrTimeout);
            return;
        }
    }
}

// ------------------------------------------------------------------ roles

// Item pacing.  Every CTA of a global-attention or SGA launch streams the
// whole K/V of one head per item, and the CTAs work on items of the same
// head at the same time; the L2 serves them all only while they read
// nearby key tiles.  Once a head's K/V is larger than the L2 (N >= ~400
// frames at H = 16), CTAs that drift apart by a fraction of an item make it
// thrash: DRAM reads grew from 0.76 TB to 2.6 TB per launch at N = 400 for
// the same work, and the power they cost lowered the clock under the power
// cap.  So a CTA's producer, before it streams its next item, waits until
// every CTA has issued the loads of the previous wave of items.  The wait
// is bounded -- by an eighth of the CTA's own last item time, at least
// kPaceLimitNs, so CTAs on the slower side of the chip (items of ~14 ms at
// N = 800) are waited for while a missing CTA costs at most 1/8 -- and falls
// through silently: pacing only orders the work in time, it never changes a
// result, and a CTA that cannot see the others (a counter shared by
// mistake, an aborted launch) just goes on.
// The pacing counters; launches take the slots in turn, and the host zeroes
// a slot on the launch's stream right before the launch.
__device__ unsigned int g_vggt_pace[kPaceSlots];

__device__ __forceinline__ unsigned int load_acquire_gpu(const unsigned int *ptr)
{
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ptr) : "memory");
    return v;
}

__device__ __forceinline__ void pace_wait(const unsigned int *pace, unsigned int target, uint64_t limit_ns)
{
    if (load_acquire_gpu(pace) >= target)
        return;
    const uint64_t t0 = globaltimer_ns();
    while (load_acquire_gpu(pace) < target && globaltimer_ns() - t0 < limit_ns)
        __nanosleep(256);
}

// kGeneral: the launch may hold split items or run in register mode.  A
// launch with neither (global attention or SGA with an even number of query
// tiles per head) uses the lean instantiation, whose issuer carries no
// split bookkeeping: its single thread shares a sub-partition with two
// softmax warps, and every instruction of it shows in the step time.
template <bool kGeneral>
__device__ __forceinline__ void run_producer(AttnSmem &sm, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                             const CUtensorMap *tmV, const AttnParams &p, int my_items)
{
    // The whole warp runs this loop (so every operand is warp-uniform); one
    // elected lane issues the copies.
    volatile WaitCtl *ab = &sm.ctl;
    const bool leader = elect_one();
    uint32_t q_issued = 0, k_issued = 0, v_issued = 0;
    uint64_t pace_limit = kPaceLimitNs, item_t0 = 0;  // pacing bound; start of the current item
    // bytes one tile load delivers: a register-mode box holds n_special * F rows
    const uint32_t tile_bytes =
        (kGeneral && p.mode == kModeRegister) ? static_cast<uint32_t>(p.tile_rows) * kHeadDim * 2 : kTileBytes;
    for (int it = 0; it < my_items; ++it) {
        const ItemWork iw = item_work(p, blockIdx.x + it * gridDim.x);
        const int qb = it & 1;
        if (p.pace && leader) {
            if (it > 0) {
                const uint64_t now = globaltimer_ns();
                const uint64_t eighth = (now - item_t0) / 8;
                pace_limit = eighth > kPaceLimitNs ? eighth : kPaceLimitNs;
                pace_wait(p.pace, static_cast<unsigned int>(it) * gridDim.x, pace_limit);  // items 0 .. it-1 streamed
            }
            item_t0 = globaltimer_ns();
        }
        __syncwarp();
        if (!wait_bar_warp(smem_u32(&sm.q_empty[qb]), ((it >> 1) & 1) ^ 1, ab, kSiteQEmpty))
            goto out;
        if (leader) {
            mbar_arrive_expect_tx(smem_u32(&sm.q_full[qb]), 2 * tile_bytes);
            for (int g = 0; g < 2; ++g) {
                if (kGeneral && p.mode == kModeRegister)  // tile q0 / 128 = frames [F t, F t + F)
                    tma_load_4d(smem_u32(sm.q[qb][g]), tmQ, smem_u32(&sm.q_full[qb]), 0, iw.w[g].h, 0,
                                (iw.w[g].q0 / kBlockM) * p.tile_frames);
                else
                    tma_load_3d(smem_u32(sm.q[qb][g]), tmQ, smem_u32(&sm.q_full[qb]), 0, iw.w[g].h, iw.w[g].q0);
            }
        }
        ++q_issued;
        // One K/V stream for the pair, or (split) one per warpgroup, in
        // step order: warpgroup 0's tile, then warpgroup 1's.
        const int streams = (kGeneral && iw.split) ? 2 : 1;
        for (int j = 0; j < p.n_kt; ++j) {
            for (int g = 0; g < streams; ++g) {
                const Work &w = iw.w[g];
                const uint32_t u = k_issued;
                const uint32_t st = u % kStages, ph = ((u / kStages) & 1) ^ 1;
                if (!wait_bar_warp(smem_u32(&sm.k_empty[st]), ph, ab, kSiteKEmpty))
                    goto out;
                if (leader) {
                    mbar_arrive_expect_tx(smem_u32(&sm.k_full[st]), tile_bytes);
                    if (kGeneral && p.mode == kModeRegister)
                        tma_load_4d(smem_u32(sm.k[st]), tmK, smem_u32(&sm.k_full[st]), 0, w.h, 0, j * p.tile_frames);
                    else
                        tma_load_3d(smem_u32(sm.k[st]), tmK, smem_u32(&sm.k_full[st]), 0, w.h, w.key0 + j * kBlockN);
                }
                ++k_issued;
                if (!wait_bar_warp(smem_u32(&sm.v_empty[st]), ph, ab, kSiteVEmpty))
                    goto out;
                if (leader) {
                    mbar_arrive_expect_tx(smem_u32(&sm.v_full[st]), tile_bytes);
                    if (kGeneral && p.mode == kModeRegister)
                        tma_load_4d(smem_u32(sm.v[st]), tmV, smem_u32(&sm.v_full[st]), 0, w.h, 0, j * p.tile_frames);
                    else
                        tma_load_3d(smem_u32(sm.v[st]), tmV, smem_u32(&sm.v_full[st]), 0, w.h, w.key0 + j * kBlockN);
                }
                ++v_issued;
            }
        }
        if (p.pace && leader)
            atomicAdd(p.pace, 1u);  // this CTA's loads of item `it` are issued
    }
out:
    // Every copy this warp started must land before the CTA may exit.
    if (leader) {
        for (uint32_t u = (k_issued > kStages ? k_issued - kStages : 0); u < k_issued; ++u)
            wait_drain(smem_u32(&sm.k_full[u % kStages]), (u / kStages) & 1);
        for (uint32_t u = (v_issued > kStages ? v_issued - kStages : 0); u < v_issued; ++u)
            wait_drain(smem_u32(&sm.v_full[u % kStages]), (u / kStages) & 1);
        for (uint32_t u = (q_issued > 2 ? q_issued - 2 : 0); u < q_issued; ++u)
            wait_drain(smem_u32(&sm.q_full[u & 1]), (u >> 1) & 1);
    }
    __syncwarp();
}

// Position of one step k in the issue order (warpgroup k & 1, key tile
// k >> 1), advanced incrementally so the issuing thread divides only once
// per item.  The K/V ring stage advances after warpgroup 1's step of a
// shared stream and after every step of a split item.
struct StepCursor {
    int k;         // step
    int j;         // key tile within the item
    int it;        // item (of this CTA)
    uint32_t st;   // K/V ring stage of the step's tile
    uint32_t ph;   // phase of that stage
    uint32_t buf;  // score buffer k % 3
    bool split;    // the item streams K/V per warpgroup

    template <bool kGeneral>
    __device__ __forceinline__ void next(const AttnParams &p)
    {
        const bool adv = (kGeneral && split) || (k & 1);
        if (k & 1) {
            if (++j == p.n_kt) {
                j = 0;
                ++it;
                if (kGeneral)
                    split = item_split(p, static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x));
            }
        }
        if (adv && ++st == kStages) {
            st = 0;
            ph ^= 1u;
        }
        ++k;
        buf = (buf == kScoreBufs - 1) ? 0u : buf + 1;
    }
};

// Shared-memory descriptors of the first Q, K and V tiles; the others are
// whole 16 KB tiles further on (kTileBytes >> 4 in the address field).
struct TileDescs {
    uint64_t q0, k0, v0;
};
constexpr uint64_t kTileDescStep = kTileBytes >> 4;

// Operands and follow-up commits of one S = Q K^T group (step k: warpgroup
// k & 1, key tile k >> 1, score buffer k % 3).  K-major operands, 128-byte
// swizzle: 8-row groups 1024 B apart, K16 step = +32 B (+2 in the
// descriptor).  Warpgroup 1's S is the last reader of a shared K tile (and,
// on the last tile of an item, of Q); in a split item each S is the only
// reader of its K tile.
struct ScoreOps {
    uint64_t a, b;
    uint32_t d;
    uint32_t bar_full;   // s_full of the buffer, 0 = do not signal
    uint32_t bar_k;      // k_empty of the stage, 0 = not the last reader
    uint32_t bar_q;      // q_empty of the buffer, 0 = not the last reader
};

template <bool kGeneral>
__device__ __forceinline__ ScoreOps score_ops(AttnSmem &sm, uint32_t tmem, const AttnParams &p, const StepCursor &s,
                                              const TileDescs &td)
{
    const uint32_t wg = static_cast<uint32_t>(s.k) & 1u;
    const uint32_t qb = static_cast<uint32_t>(s.it) & 1u;
    ScoreOps o;
    o.a = td.q0 + (2 * qb + wg) * kTileDescStep;
    o.b = td.k0 + s.st * kTileDescStep;
    o.d = tmem + s.buf * kBlockN;
    o.bar_full = (p.stall_first_scores && s.k == 0) ? 0u : smem_u32(&sm.s_full[s.buf]);
    o.bar_k = (wg || (kGeneral && s.split)) ? smem_u32(&sm.k_empty[s.st]) : 0u;
    o.bar_q = (wg && s.j == p.n_kt - 1) ? smem_u32(&sm.q_empty[qb]) : 0u;
    return o;
}

// Waits until the Q and K tiles of step s have landed (warpgroup 0's S is
// the first reader of the item's Q tiles and of a shared K tile).
template <bool kGeneral>
__device__ __forceinline__ bool score_inputs_ready(AttnSmem &sm, const StepCursor &s, volatile WaitCtl *ab)
{
    const bool wg1 = (s.k & 1) != 0;
    if (wg1 && !(kGeneral && s.split))
        return true;
    if (!wg1 && s.j == 0 &&
        !wait_bar(smem_u32(&sm.q_full[s.it & 1]), (static_cast<uint32_t>(s.it) >> 1) & 1u, ab, kSiteQFull))
        return false;
    return wait_bar(smem_u32(&sm.k_full[s.st]), s.ph, ab, kSiteKFull);
}

__device__ __forceinline__ void issue_score_ops(const ScoreOps &o)
{
    constexpr uint32_t kIdescS = idesc_bf16_f32(kBlockM, kBlockN, false);
#pragma unroll
    for (int kk = 0; kk < kHeadDim / 16; ++kk)
        umma_ss(o.d, o.a + 2 * kk, o.b + 2 * kk, kIdescS, kk > 0 ? 1u : 0u);
    if (o.bar_full)
        umma_commit(o.bar_full);
    if (o.bar_k)
        umma_commit(o.bar_k);
    if (o.bar_q)
        umma_commit(o.bar_q);
}

// Keeps values computed before the next volatile asm (a barrier wait).
__device__ __forceinline__ void hold(const ScoreOps &o)
{
    asm volatile("" ::"l"(o.a), "l"(o.b), "r"(o.d), "r"(o.bar_full), "r"(o.bar_k), "r"(o.bar_q));
}

// O += P V for step k.  V is an MN-major B operand: the 64 head-dim values
// of a key are one 128-byte swizzled row, 8-key groups 1024 B apart, K16
// step = 2048 B (+128).  P: bf16 pairs in the first 64 columns of the score
// buffer, 8 columns per K16 step.
template <bool kGeneral>
__device__ __forceinline__ void issue_pv(AttnSmem &sm, uint32_t tmem, const AttnParams &p, const StepCursor &v,
                                         const TileDescs &td)
{
    constexpr uint32_t kIdescPV = idesc_bf16_f32(kBlockM, kHeadDim, true);
    const int wg = v.k & 1;
    const uint64_t b = td.v0 + v.st * kTileDescStep;
    const uint32_t d = tmem + kTmemO + static_cast<uint32_t>(wg * kHeadDim);
    const uint32_t a = tmem + v.buf * kBlockN;
#pragma unroll
    for (int kk = 0; kk < kBlockN / 16; ++kk)
        umma_ts(d, a + 8 * kk, b + 128 * kk, kIdescPV, (v.j > 0 || kk > 0) ? 1u : 0u);
    umma_commit(smem_u32(&sm.o_done[wg]));
    if (v.j == p.n_kt - 1)
        umma_commit(smem_u32(&sm.o_final[wg]));
    if (wg == 1 || (kGeneral && v.split))
        umma_commit(smem_u32(&sm.v_empty[v.st]));
}

// The issuer runs on one thread: its scalar code shares a sub-partition
// with two busy softmax warps, and every cycle between UMMA groups can
// leave the tensor pipe idle.  So the wait for PV(k) (about 500 cycles)
// absorbs the bookkeeping and the operands of S(k + 3), which then issues
// right after it.
template <bool kGeneral>
__device__ __forceinline__ void mma_loop(AttnSmem &sm, uint32_t tmem, const AttnParams &p, int total_tiles,
                                         volatile WaitCtl *ab)
{
    const int steps = 2 * total_tiles;
    const TileDescs td{sdesc_sw128(smem_u32(sm.q[0][0]), 16, 1024), sdesc_sw128(smem_u32(sm.k[0]), 16, 1024),
                       sdesc_sw128(smem_u32(sm.v[0]), 16, 1024)};
    const bool split0 = kGeneral && item_split(p, static_cast<int>(blockIdx.x));
    StepCursor s{0, 0, 0, 0u, 0u, 0u, split0};  // next S to issue
    StepCursor v{0, 0, 0, 0u, 0u, 0u, split0};  // next PV to issue
    for (; s.k < steps && s.k < kScoreBufs; s.next<kGeneral>(p)) {
        const ScoreOps so = score_ops<kGeneral>(sm, tmem, p, s, td);
        if (!score_inputs_ready<kGeneral>(sm, s, ab))
            return;
        tc_fence_after();
        issue_score_ops(so);
    }
    while (v.k < steps) {
        const int wg = v.k & 1;
        const uint32_t cpar = static_cast<uint32_t>(v.k >> 1) & 1u;
        if ((wg == 0 || (kGeneral && v.split)) && !wait_bar(smem_u32(&sm.v_full[v.st]), v.ph, ab, kSiteVFull))
            return;
        // p_ready[wg][c & 1], phase c >> 1 (c = v.k >> 1): see run_softmax.
        if (!wait_bar(smem_u32(&sm.p_ready[wg][cpar]), (static_cast<uint32_t>(v.k) >> 2) & 1u, ab, kSitePReady))
            return;
        tc_fence_after();
        issue_pv<kGeneral>(sm, tmem, p, v, td);
        v.next<kGeneral>(p);
        if (s.k < steps) {
            // S(k + 3) overwrites the buffer PV(k) reads P from.
            const ScoreOps so = score_ops<kGeneral>(sm, tmem, p, s, td);
            if (!score_inputs_ready<kGeneral>(sm, s, ab))
                return;
            s.next<kGeneral>(p);
            hold(so);
            if (!wait_bar(smem_u32(&sm.o_done[wg]), cpar, ab, kSiteODone))
                return;
            tc_fence_after();
            issue_score_ops(so);
        }
    }
}

template <bool kGeneral>
__device__ __forceinline__ void run_mma(AttnSmem &sm, uint32_t tmem, const AttnParams &p, int total_tiles)
{
    volatile WaitCtl *ab = &sm.ctl;
    if (elect_one()) {
        mma_loop<kGeneral>(sm, tmem, p, total_tiles, ab);
        // Every UMMA issued must complete before TMEM is released.
        umma_commit(smem_u32(&sm.drain));
        wait_drain(smem_u32(&sm.drain), 0);
    }
    __syncwarp();
}

__device__ __forceinline__ float dot64_bf16(const uint4 *a, const uint4 *b)
{
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 x = __ldg(a + i), y = __ldg(b + i);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16lo_to_f32(xs[e]), bf16lo_to_f32(ys[e]), acc);
            acc = fmaf(bf16hi_to_f32(xs[e]), bf16hi_to_f32(ys[e]), acc);
        }
    }
    return acc;
}

__device__ __forceinline__ float dot64_bf16_f32(const uint4 *a, const float *b)
{
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 x = __ldg(a + i);
        const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc = fmaf(bf16lo_to_f32(xs[e]), __ldg(b + 8 * i + 2 * e), acc);
            acc = fmaf(bf16hi_to_f32(xs[e]), __ldg(b + 8 * i + 2 * e + 1), acc);
        }
    }
    return acc;
}

// The end of an item for one query row without the SGA terms: O (64 fp32
// columns of this warpgroup's accumulator) divided by l, stored as bf16,
// and lse.  The caller has waited for the item's last PV.
__device__ __forceinline__ void finish_row(const AttnParams &p, uint32_t tO, int row, bool row_ok, int h, float l,
                                           float m)
{
    uint32_t o[2][32];
    tmem_ld32(tO, o[0]);
    tmem_ld32(tO + 32, o[1]);
    tmem_ld_wait();
    reg_fence(o[0]);
    reg_fence(o[1]);
    if (row_ok && VGGT_IN_RANGE(row >= 0 && row < (p.mode == kModeRegister ? p.n_frames * p.L : p.S) && h < p.H,
                                kCheckAttnRow)) {
        const float inv = 1.f / l;
        uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(row) * p.H + h) * kHeadDim);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint32_t wv[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int cc = 8 * i + 2 * e;
                wv[e] = pack_bf16x2(__uint_as_float(o[cc >> 5][cc & 31]) * inv,
                                    __uint_as_float(o[(cc + 1) >> 5][(cc + 1) & 31]) * inv);
            }
            orow[i] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        if (p.lse)
            p.lse[static_cast<size_t>(row) * p.H + h] = (m + __log2f(l)) * 0.69314718055994531f;
    }
}

template <bool kGeneral>
__device__ __forceinline__ void run_softmax(AttnSmem &sm, uint32_t tmem, const AttnParams &p, int my_items,
                                            int wg)
{
    volatile WaitCtl *ab = &sm.ctl;
    const int t = static_cast<int>(threadIdx.x) - kBlockM * (wg + 1);  // row within the tile
    const uint32_t lane_off = static_cast<uint32_t>((t >> 5) * 32) << 16;
    const uint32_t tO = tmem + kTmemO + static_cast<uint32_t>(wg * kHeadDim) + lane_off;
    const uint32_t bar_s0 = smem_u32(&sm.s_full[0]);
    // The four warps of a warpgroup meet only through the barriers, and
    // S(k + 2) is issued before every warp has finished step k, so one warp
    // can start its next step while another is still on this one.  Its
    // arrival must not count towards the step it has left: the two P-ready
    // barriers of a warpgroup alternate by step (no warp is ever two steps
    // ahead, since S(k + 4) needs all of step k).
    const uint32_t bar_p0 = smem_u32(&sm.p_ready[wg][0]);
    const uint32_t bar_o = smem_u32(&sm.o_done[wg]);
    const uint32_t bar_of = smem_u32(&sm.o_final[wg]);
    const float sl2 = p.scale_log2;
    const uint64_t sl2_2 = f2_pack(sl2, sl2);
    const uint64_t magic2 = f2_pack(kRoundMagic, kRoundMagic);
    const uint64_t neg_magic2 = f2_pack(-kRoundMagic, -kRoundMagic);
    const uint64_t neg_one2 = f2_pack(-1.f, -1.f);
    const uint64_t c0_2 = f2_pack(kExp2C0, kExp2C0), c1_2 = f2_pack(kExp2C1, kExp2C1);
    const uint64_t c2_2 = f2_pack(kExp2C2, kExp2C2), c3_2 = f2_pack(kExp2C3, kExp2C3);
    uint32_t c = 0, o_seen = 0;
    // The general instantiation (frame and register launches, split items)
    // defers an item's epilogue into the next item's first step, after its
    // P is stored and before its P-ready arrive: the wait for the item's
    // last PV then hides behind a whole softmax step, where it would
    // otherwise idle both warpgroups at every item end (11 key tiles per
    // item in frame mode).  SGA keeps its in-place epilogue (diagonal and
    // mean terms).
    const bool defer = kGeneral && p.mode != kModeSga;
    int prev_row = 0, prev_h = 0;
    bool prev_ok = false;
    float prev_l = 1.f, prev_m = 0.f;

    for (int it = 0; it < my_items; ++it) {
        const Work w = wg_work(p, blockIdx.x + it * gridDim.x, wg);
        int row = w.q0 + t;
        bool row_ok = row < w.row_end;
        if (kGeneral && p.mode == kModeRegister) {
            // tile row r = (frame in the tile, special token) -> token frame * L + slot
            const int r = row % kBlockM, fr = r / p.n_special;
            const int frame = (row / kBlockM) * p.tile_frames + fr, slot = r - fr * p.n_special;
            row_ok = row_ok && r < p.tile_rows && frame < p.n_frames;
            row = frame * p.L + slot;
        }

        // SGA: diagonal logit (query's own key, when it was dropped) and the
        // mean-column logit q.kbar*scale + ln M, both in log2 units.
        float diag_l2 = -INFINITY, mean_l2 = -INFINITY;
        if (p.mode == kModeSga && row_ok && VGGT_IN_RANGE(row < p.S && w.h < p.H, kCheckSgaSeed)) {
            const int Mi = __ldg(p.mult + p.row0 + row);
            const size_t off = (static_cast<size_t>(row) * p.H + w.h) * kHeadDim;
            const size_t own = (static_cast<size_t>(p.own_row0 + row) * p.H + w.h) * kHeadDim;
            const uint4 *qr = reinterpret_cast<const uint4 *>(p.q + off);
            if (p.n_dropped > 0 && Mi == p.n_dropped - 1)
                diag_l2 = dot64_bf16(qr, reinterpret_cast<const uint4 *>(p.k + own)) * sl2;
            if (Mi > 0)
                mean_l2 = fmaf(dot64_bf16_f32(qr, p.kbar + w.h * kHeadDim), sl2, __log2f(static_cast<float>(Mi)));
        }
        float m = fmaxf(diag_l2, mean_l2);
        float l = 0.f;

        for (int j = 0; j < p.n_kt; ++j, ++c) {
            // Step k = 2c + wg uses score buffer k % 3 (its (k / 3)-th use).
            const uint32_t k = 2 * c + static_cast<uint32_t>(wg);
            const uint32_t buf = k % kScoreBufs;
            const uint32_t tS = tmem + buf * kBlockN + lane_off;
            if (!wait_bar_warp(bar_s0 + 8 * buf, (k / kScoreBufs) & 1, ab, kSiteSFull))
                return;
            tc_fence_after();
            uint32_t s[4][32];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                tmem_ld32(tS + 32 * i, s[i]);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 4; ++i)
                reg_fence(s[i]);

            // register mode: key tile j holds frames [F j, F j + F), the first
            // n_special * (frames present) columns of it
            const int valid = (kGeneral && p.mode == kModeRegister)
                                  ? min(p.tile_rows, (p.n_frames - j * p.tile_frames) * p.n_special)
                                  : w.n_keys - j * kBlockN;
            auto mask_tail = [&]() {
                if (valid < kBlockN) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            if (32 * i + e >= valid)
                                s[i][e] = __float_as_uint(-INFINITY);
                }
            };
            mask_tail();
            // Row max of the tile, in log2 units.
            auto tile_max = [&]() -> float {
                float mx[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    mx[i] = fmax3(__uint_as_float(s[i][0]), __uint_as_float(s[i][1]), __uint_as_float(s[i][2]));
#pragma unroll
                    for (int e = 3; e < 31; e += 2)
                        mx[i] = fmax3(mx[i], __uint_as_float(s[i][e]), __uint_as_float(s[i][e + 1]));
                    mx[i] = fmaxf(mx[i], __uint_as_float(s[i][31]));
                }
                return fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
            };
            // P = 2^(s*scale*log2e - m), packed to bf16 pairs in pk and stored
            // over the first 64 columns of the score buffer; returns the
            // row's sum of the tile's P (fp32, before rounding to bf16).  The
            // lean instantiation stores each 32-column chunk as soon as it is
            // packed (the stores overlap the next chunk's exponentials) and
            // keeps S in registers for the slow path below; the general one
            // stores P only once the tile is accepted and reads S back from
            // the score buffer in the slow path (fewer live registers: with
            // S live its loop spills).
            constexpr bool kStoreEarly = !kGeneral;
            uint32_t pk[4][16];
            auto exp_tile = [&]() -> float {
                const uint64_t neg_m2 = f2_pack(-m, -m);
                uint64_t ls[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const uint64_t x2 = f2_fma(
                            f2_pack(__uint_as_float(s[i][2 * e]), __uint_as_float(s[i][2 * e + 1])), sl2_2, neg_m2);
                        float a, b;
                        f2_unpack(x2, a, b);
                        if (e < kExp2PolyPairs) {
                            const uint64_t xc = f2_pack(fmaxf(a, kExp2MinArg), fmaxf(b, kExp2MinArg));
                            const uint64_t y = f2_add(xc, magic2);       // round(x) in the low mantissa bits
                            const uint64_t jj = f2_add(y, neg_magic2);   // round(x) as a float
                            const uint64_t f = f2_fma(jj, neg_one2, xc); // x - j, in [-1/2, 1/2]
                            uint64_t q = f2_fma(c3_2, f, c2_2);
                            q = f2_fma(q, f, c1_2);
                            q = f2_fma(q, f, c0_2);
                            float qa, qb, ya, yb;
                            f2_unpack(q, qa, qb);
                            f2_unpack(y, ya, yb);
                            a = __uint_as_float(__float_as_uint(ya) * 8388608u + __float_as_uint(qa));
                            b = __uint_as_float(__float_as_uint(yb) * 8388608u + __float_as_uint(qb));
                        } else {
                            a = ex2_approx(a);
                            b = ex2_approx(b);
                        }
                        ls[e & 3] = f2_add(ls[e & 3], f2_pack(a, b));
                        pk[i][e] = pack_bf16x2(a, b);
                    }
                    if constexpr (kStoreEarly)
                        tmem_st16(tS + 16 * i, pk[i]);
                }
                const uint64_t t2 = f2_add(f2_add(ls[0], ls[1]), f2_add(ls[2], ls[3]));
                float ta, tb;
                f2_unpack(t2, ta, tb);
                return ta + tb;
            };

            // Lazy offset: the first tile of an item sets m to its row max;
            // later tiles are exponentiated against the current m without
            // computing their max.  A row whose tile sum exceeds
            // kTileSumLimit (so some P of it may exceed kTileSumLimit) makes
            // the warp take the slow path: the tile max (from S in registers,
            // or read back from the score buffer, which P has not yet
            // overwritten), a rescale of O and l for the rows whose max grew
            // by more than kRescaleThreshold, and the tile's P again.  P stays
            // below 2^15 (bf16 and the fp32 accumulators have the range) and
            // is read by the issuer only after this step's P-ready arrive, so
            // it may be written twice.
            if (j == 0)
                m = fmaxf(m, tile_max());
            float tsum = exp_tile();
            if (j > 0 && __any_sync(0xffffffffu, !(tsum <= kTileSumLimit))) {
                if constexpr (!kStoreEarly) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        tmem_ld32(tS + 32 * i, s[i]);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        reg_fence(s[i]);
                    mask_tail();
                }
                const float cand = tile_max();
                const bool need = cand > m + kRescaleThreshold;
                if (__any_sync(0xffffffffu, need)) {
                    // O may be touched only after PV(c-1) has completed.  S(k)
                    // was issued after PV(c-2) completed, so the o_done phase
                    // of PV(c-1) is the current or the last one: its parity
                    // is unambiguous.
                    if (o_seen < c) {
                        if (!wait_bar_warp(bar_o, (c - 1) & 1, ab, kSiteODone))
                            return;
                        o_seen = c;
                    }
                    tc_fence_after();
                    const float f = need ? ex2_approx(m - cand) : 1.f;
                    // 16 columns at a time: S is still live in registers
#pragma unroll 1
                    for (int quarter = 0; quarter < 4; ++quarter) {
                        uint32_t o[16];
                        tmem_ld16(tO + 16 * quarter, o);
                        tmem_ld_wait();
                        reg_fence(o);
#pragma unroll
                        for (int e = 0; e < 16; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
                        tmem_st16(tO + 16 * quarter, o);
                    }
                    tmem_st_wait();
                    if (need) {
                        l *= f;
                        m = cand;
                    }
                }
                // The tile's P again, against the new offset.
                if constexpr (kStoreEarly)
                    tmem_st_wait();  // the first pass's P stores land before they are overwritten
                tsum = exp_tile();
            }
            if constexpr (!kStoreEarly) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    tmem_st16(tS + 16 * i, pk[i]);
            }
            l += tsum;
            tmem_st_wait();
            if (kGeneral && defer && j == 0 && it > 0) {
                // the previous item's epilogue: its PVs precede this P-ready
                if (!wait_bar_warp(bar_of, static_cast<uint32_t>(it - 1) & 1, ab, kSiteOFinal))
                    return;
                o_seen = c;
                tc_fence_after();
                finish_row(p, tO, prev_row, prev_ok, prev_h, prev_l, prev_m);
            }
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0)
                mbar_arrive(bar_p0 + 8 * (c & 1));
        }

        if (kGeneral && defer) {
            prev_row = row;
            prev_ok = row_ok;
            prev_h = w.h;
            prev_l = l;
            prev_m = m;
            continue;
        }

        // Epilogue: every PV of this item must have completed.  Up to two of
        // them can still be in flight here, which the o_done parity cannot
        // tell apart, so the issuer signals the item's last PV on o_final.
        if (!wait_bar_warp(bar_of, static_cast<uint32_t>(it) & 1, ab, kSiteOFinal))
            return;
        o_seen = c;
        tc_fence_after();
        uint32_t o[2][32];
        tmem_ld32(tO, o[0]);
        tmem_ld32(tO + 32, o[1]);
        tmem_ld_wait();
        reg_fence(o[0]);
        reg_fence(o[1]);
        tc_fence_before();

        float ltot = l;
        if (p.mode == kModeSga && row_ok) {
            const float wd = (diag_l2 > -INFINITY) ? ex2_approx(diag_l2 - m) : 0.f;
            const float wm = (mean_l2 > -INFINITY) ? ex2_approx(mean_l2 - m) : 0.f;
            ltot += wd + wm;
            const size_t own = (static_cast<size_t>(p.own_row0 + row) * p.H + w.h) * kHeadDim;
            const uint4 *vr = reinterpret_cast<const uint4 *>(p.v + own);
            const float *vb = p.vbar + w.h * kHeadDim;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint4 x = (wd != 0.f) ? __ldg(vr + i) : make_uint4(0, 0, 0, 0);
                const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int cc = 8 * i + 2 * e;
                    float lo = __uint_as_float(o[cc >> 5][cc & 31]);
                    float hi = __uint_as_float(o[(cc + 1) >> 5][(cc + 1) & 31]);
                    lo = fmaf(wd, bf16lo_to_f32(xs[e]), lo);
                    hi = fmaf(wd, bf16hi_to_f32(xs[e]), hi);
                    if (wm != 0.f) {
                        lo = fmaf(wm, __ldg(vb + cc), lo);
                        hi = fmaf(wm, __ldg(vb + cc + 1), hi);
                    }
                    o[cc >> 5][cc & 31] = __float_as_uint(lo);
                    o[(cc + 1) >> 5][(cc + 1) & 31] = __float_as_uint(hi);
                }
            }
        }
        if (row_ok && VGGT_IN_RANGE(row >= 0 && row < (p.mode == kModeRegister ? p.n_frames * p.L : p.S) && w.h < p.H,
                                    kCheckAttnRow)) {
            const float inv = 1.f / ltot;
            uint4 *orow = reinterpret_cast<uint4 *>(p.o + (static_cast<size_t>(row) * p.H + w.h) * kHeadDim);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t wv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int cc = 8 * i + 2 * e;
                    wv[e] = pack_bf16x2(__uint_as_float(o[cc >> 5][cc & 31]) * inv,
                                        __uint_as_float(o[(cc + 1) >> 5][(cc + 1) & 31]) * inv);
                }
                orow[i] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            if (p.lse)
                p.lse[static_cast<size_t>(row) * p.H + w.h] = (m + __log2f(ltot)) * 0.69314718055994531f;
        }
    }
    if (kGeneral && defer && my_items > 0) {
        if (!wait_bar_warp(bar_of, static_cast<uint32_t>(my_items - 1) & 1, ab, kSiteOFinal))
            return;
        tc_fence_after();
        finish_row(p, tO, prev_row, prev_ok, prev_h, prev_l, prev_m);
        tc_fence_before();
    }
}

template <bool kGeneral>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p)
{
    extern __shared__ uint8_t smem_raw[];
    AttnSmem &sm = *reinterpret_cast<AttnSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int my_items =
        (p.n_items > static_cast<int>(blockIdx.x)) ? (p.n_items - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < kScoreBufs; ++i)
            mbar_init(smem_u32(&sm.s_full[i]), 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.q_full[i]), 1);
            mbar_init(smem_u32(&sm.q_empty[i]), 1);
            mbar_init(smem_u32(&sm.p_ready[i][0]), 4);
            mbar_init(smem_u32(&sm.p_ready[i][1]), 4);
            mbar_init(smem_u32(&sm.o_done[i]), 1);
            mbar_init(smem_u32(&sm.o_final[i]), 1);
        }
        for (int i = 0; i < kStages; ++i) {
            mbar_init(smem_u32(&sm.k_full[i]), 1);
            mbar_init(smem_u32(&sm.k_empty[i]), 1);
            mbar_init(smem_u32(&sm.v_full[i]), 1);
            mbar_init(smem_u32(&sm.v_empty[i]), 1);
        }
        mbar_init(smem_u32(&sm.drain), 1);
        sm.ctl.abort = 0;
        sm.ctl.limit_ns = p.wait_limit_ns;
        fence_mbar_init();
        fence_proxy_async_smem();
    }
    if (kGeneral && p.mode == kModeRegister && p.tile_rows < kBlockM) {
        // Register mode loads n_special * F rows per tile; the rows after
        // them are never written by TMA.  Zero them in every Q, K and V
        // buffer once, so the UMMAs read finite values there (masked keys
        // get P = 0, which must not meet a NaN in V).
        const int tail = (kBlockM - p.tile_rows) * kHeadDim * 2 / 16;  // uint4 per tile
        constexpr int kTiles = 4 + 2 * kStages;
        for (int i = threadIdx.x; i < kTiles * tail; i += blockDim.x) {
            const int t = i / tail, e = i - t * tail;
            uint8_t *base = t < 4 ? sm.q[t >> 1][t & 1] : (t < 4 + kStages ? sm.k[t - 4] : sm.v[t - 4 - kStages]);
            reinterpret_cast<uint4 *>(base + p.tile_rows * kHeadDim * 2)[e] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmK);
        prefetch_tensormap(&tmV);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    // Launched at 168 registers/thread (384 x 168 = 64512): the control
    // warpgroup drops to 72 and the two softmax warpgroups rise to 216,
    // 128 x (72 + 216 + 216) = 64512, so the increases are always covered.
    if (warp < 4) {
        setmaxnreg_dec<kRegsControl>();
        if (warp == 0)
            run_producer<kGeneral>(sm, &tmQ, &tmK, &tmV, p, my_items);
        else if (warp == 1)
            run_mma<kGeneral>(sm, tmem, p, my_items * p.n_kt);
    } else {
        setmaxnreg_inc<kRegsSoftmax>();
        run_softmax<kGeneral>(sm, tmem, p, my_items, (warp >> 2) - 1);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

} // namespace vggt
