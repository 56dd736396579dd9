// prefill_tc.cu -- causal prefill attention over the paged pool with deferred
// RoPE on the fifth-generation tensor cores (tcgen05.mma, accumulators in
// tensor memory, K/V tiles staged by TMA).
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Prefilling -- the kernel reads the cached KV blocks and
// rotates once, by the distance from the cached document's offset to the
// query's position, rather than taking the keys back to position 0 and
// rotating them a second time; this phase is bound by compute.
//
// Where the single relative rotation goes.  Keys sit in the pool rotated at
// their local index j.  Each CTA fixes a reference position P0 (its first
// query token's position) and rotates its query tile once, Q'_i =
// R(p_i - P0) q_i.  Every K tile, after TMA has landed it in shared memory,
// gets one relative rotation R(o - P0) by its segment's offset o -- not a
// reset to position 0 followed by a second rotation -- so that scores carry
// the angle (p_i - o - j) of eager RoPE attention.  The rotation runs two
// stages ahead of the MMAs that read the tile.  The plain (materialised)
// path is the same kernel with that rotation removed: keys arrive rotated
// at their absolute positions and the query is rotated at p_i.
//
// CTA = 256 query rows (two 128-row MMA tiles) of one KV head of one
// request; rows are (token, head-in-group) pairs, token-major, so each K/V
// tile loaded by TMA serves every query head of its group and both row
// tiles.  16 warps in four warpgroups, registers rebalanced with setmaxnreg
// (producers/MMA 72, softmax 192, K rotation 56 per thread):
//   warp 0      K producer: walks the table once, publishes per-tile
//               information (blocks, metadata, mask flag) in a shared-memory
//               ring, and TMA-loads K tiles (<= 8 blocks = 128 keys of one
//               segment) into 3 stages -- two 16 KiB boxes when the tile's
//               blocks are consecutive in the pool, else two 2 KiB boxes per
//               block
//   warp 1      V producer: the same for V tiles, 2 stages
//   warp 2      MMA issuer for both row tiles, in ping-pong order (and owner of
//               tensor memory); warp 3 has no role
//   warps 4-7   row tile 0, one thread per row: first the rotated query rows
//               of the tile, then per K tile the online softmax with the whole
//               128-column score row in registers (one tensor-memory load,
//               mask, max, 2^(S - m), one store of P over the consumed S
//               columns), lazy rescaling of O; epilogue O / l
//   warps 8-11  the same for row tile 1
//   warps 12-15 K rotation: every K tile once, in shared memory
// Tensor memory (512 columns): S0 [0,128) (P0 = its first 64 columns),
// S1 [128,256) (P1), O0 [256,384), O1 [384,512).
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lazy {

namespace {

constexpr int kTileRows = 128;
constexpr int kRows = 2 * kTileRows;
constexpr int kTileBlocks = 8;
constexpr int kTileBytes = kTileRows * kHeadDim * 2;   // 32 KiB
constexpr int kHalfPlane = kTileBytes / 2;             // 16 KiB
constexpr int kKStages = 3, kVStages = 2, kInfoStages = 8;
constexpr int kThreads = 512;

struct TileInfo {
    uint32_t blk[kTileBlocks];
    uint32_t meta[kTileBlocks];
    int n;       // blocks in the tile (1..8)
    int off;     // the segment's logical offset
    int flags;   // kFull: every key of the tile is visible to every row of the CTA
    int pad;
};
constexpr int kFull = 1;

constexpr int kOffQ = 0;                                     // 2 row tiles
constexpr int kOffK = kOffQ + 2 * kTileBytes;                // 3 stages
constexpr int kOffV = kOffK + kKStages * kTileBytes;         // 2 stages
constexpr int kOffInfo = kOffV + kVStages * kTileBytes;
constexpr int kOffBar = kOffInfo + kInfoStages * static_cast<int>(sizeof(TileInfo));
// barriers
constexpr int B_KFULL = 0, B_KEMPTY = B_KFULL + kKStages, B_KROT = B_KEMPTY + kKStages,
              B_VFULL = B_KROT + kKStages, B_VEMPTY = B_VFULL + kVStages, B_IFULL = B_VEMPTY + kVStages,
              B_IEMPTY = B_IFULL + kInfoStages, B_SFULL = B_IEMPTY + kInfoStages, B_PFULL = B_SFULL + 2,
              B_ODONE = B_PFULL + 2, B_QFULL = B_ODONE + 2, B_DRAIN = B_QFULL + 1, kNumBars = B_DRAIN + 1;
constexpr int kOffTheta = kOffBar + kNumBars * 8;
constexpr int kOffMisc = kOffTheta + kHalfDim * 8;
constexpr int kOffSlope = kOffMisc + 16;                    // ALiBi: slopes of the group's G heads
constexpr int kSmemUse = kOffSlope + 32 * 4;
constexpr size_t kTcSmem = kSmemUse + 1024;
static_assert(kTcSmem <= 232448, "shared memory budget");
static_assert(sizeof(TileInfo) == 80, "tile info layout");

constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays below 2^8 between rescales
// consumers of one tile-info entry: 8 softmax warps, the V producer, the MMA warp, and on the
// lazy path the 4 rotation warps
constexpr int kInfoConsumers = 10;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// 4D tiled load: 8 consecutive blocks of one head, one 64-element half (16 KiB).
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int y, int h, int b,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(h), "r"(b), "r"(smem_u32(bar))
        : "memory");
}
// Same decision for every lane of the warp.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *d_status) {
    const bool ok = wait_or_abort(bar, parity, abort_flag, d_status);
    return __all_sync(0xffffffffu, ok);
}
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(N)); }
// Register split (launch: 512 threads x 128 registers): producers + MMA warpgroup, two
// softmax warpgroups, rotation warpgroup.
constexpr int kProducerRegs = 72, kSoftmaxRegs = 192, kRotRegs = 56;
static_assert(kProducerRegs * 128 + 2 * kSoftmaxRegs * 128 + kRotRegs * 128 <= 65536, "register split");
// Same decision for the 128 threads of the rotation warpgroup.
__device__ __forceinline__ bool rot_all(bool ok) {
    uint32_t any_fail;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.eq.u32 p, %1, 0;\n barrier.cta.red.or.pred q, 2, 128, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(any_fail)
        : "r"(ok ? 1u : 0u)
        : "memory");
    return any_fail == 0;
}

// MODE: kLazy (keys from the pool, each K tile rotated by (o - P0)), kPlain (keys from a
// materialised copy indexed by table position, queries rotated at absolute positions: the
// comparison path), kAlibi (keys from the pool used as stored, nothing rotated, the ALiBi
// bias slope_h * (o + j - p) added to each score before the mask).
constexpr int kLazy = 0, kPlain = 1, kAlibi = 2;

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const __grid_constant__ CUtensorMap tmK8,
                                                                 const __grid_constant__ CUtensorMap tmV8,
                                                                 const __grid_constant__ CUtensorMap tmQ,
                                                                 const AttnParams p) {
    constexpr bool PLAIN = MODE == kPlain;   // K source indexed by table position
    constexpr bool ROTK = MODE == kLazy;     // K tiles rotated in shared memory
    constexpr bool ALIBI = MODE == kAlibi;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    float *slope_s = reinterpret_cast<float *>(sm + kOffSlope);
    TileInfo *info = reinterpret_cast<TileInfo *>(sm + kOffInfo);
    double *theta_s = reinterpret_cast<double *>(sm + kOffTheta);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);

    // work unit (m-tile, KV head, request) and which part of its keys this CTA takes
    int unit = static_cast<int>(blockIdx.x), part = -1;
    if (unit >= p.pf_base) {
        const int k = unit - p.pf_base;
        unit = p.pf_base + (k >> 1);
        part = k & 1;
    }
    const int mt = unit % p.pf_mtiles, kvh = (unit / p.pf_mtiles) % p.hkv, r = unit / (p.pf_mtiles * p.hkv);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    const int q0 = p.cu_q[r];
    const int T = p.cu_q[r + 1] - q0;
    const int R0 = mt * kRows;
    if (R0 >= T * G) return;   // uniform: this tile has no rows
    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    // words this CTA walks: all of them, or the first or second half for a split unit
    const int wbeg = part == 1 ? n_words / 2 : 0, wend = part == 0 ? n_words / 2 : n_words;
    const uint32_t *tbl = p.table + wbase;
    const int pos0 = p.q_pos0[r];
    const int tok_first = R0 / G;
    const int tok_last = min(T - 1, (R0 + kRows - 1) / G);
    const int Pbase = pos0 + tok_first;   // smallest query position of the CTA

    if (threadIdx.x == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], 1);
            mbar_init(&bars[B_KROT + i], 4);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&bars[B_VFULL + i], 1);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        for (int i = 0; i < kInfoStages; ++i) {
            mbar_init(&bars[B_IFULL + i], 1);
            mbar_init(&bars[B_IEMPTY + i], kInfoConsumers + (ROTK ? 4 : 0));
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[B_SFULL + t], 1);
            mbar_init(&bars[B_PFULL + t], 4);
            mbar_init(&bars[B_ODONE + t], 1);
        }
        // the query tiles: written by the 8 softmax warps, or loaded prepared by one TMA arrival
        mbar_init(&bars[B_QFULL], p.q_prep ? 1 : 8);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        if (mt == 0 && kvh == 0 && n_words > p.max_words) set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (threadIdx.x < kHalfDim) theta_s[threadIdx.x] = p.rope.theta[threadIdx.x];
    if (ALIBI && threadIdx.x < G) slope_s[threadIdx.x] = p.alibi_log2[kvh * G + threadIdx.x];
    if (warp == 2) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp < 4) {
    setmaxnreg_dec<kProducerRegs>();
    // The producers and the MMA issuer run their loops with the whole warp (control flow and
    // loop state uniform); TMA copies, arrivals and MMAs are issued by an elected lane, or by
    // lane k for block k of a tile whose blocks are not consecutive in the pool.
    const bool leader = tc::elect_one();
    if (warp == 0) {
        // ============================================================ table walk + K producer
        if (leader) tma_prefetch_desc(&tmK);
        int issued = 0;
        for (int w = wbeg, j = 0; w < wend; ++j) {
            // the tile: up to 8 consecutive words that share one offset; lane k < 8 holds word k
            const uint32_t wl = (lane < kTileBlocks && w + lane < wend) ? tbl[w + lane] : 0xFFFFFFFFu;
            const int off = word_offset(__shfl_sync(0xffffffffu, wl, 0));
            const bool same = lane < kTileBlocks && w + lane < wend && word_offset(wl) == off;
            const int n = __ffs(~__ballot_sync(0xffffffffu, same)) - 1;   // lanes 0..n-1 share the offset
            const uint32_t b = word_block(wl);
            const bool inb = lane < n && b < static_cast<uint32_t>(p.num_blocks);
            const uint32_t mt = inb ? p.blk_meta[b] : 0u;
            if (lane < n && !inb) set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
            const bool full = n == kTileBlocks &&
                              __all_sync(0xffffffffu, lane >= n || (meta_valid(mt) == kBlockTokens &&
                                                                    off + meta_j0(mt) + kBlockTokens - 1 <= Pbase));
            // blocks consecutive in the source: two 16 KiB boxes instead of 2n small ones
            const uint32_t b0 = __shfl_sync(0xffffffffu, b, 0);
            const bool contig =
                PLAIN || __all_sync(0xffffffffu, lane >= n || (inb && b == b0 + static_cast<uint32_t>(lane)));
            // publish the tile information
            const int is = j % kInfoStages;
            if (!warp_wait(&bars[B_IEMPTY + is], ((j / kInfoStages) & 1) ^ 1, abort_flag, p.d_status)) break;
            TileInfo &ti = info[is];
            if (lane < kTileBlocks) {
                ti.blk[lane] = lane < n ? b : 0u;
                ti.meta[lane] = mt;
            }
            if (leader) {
                ti.n = n;
                ti.off = off;
                ti.flags = full ? kFull : 0;
            }
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_IFULL + is]);
            // K tile
            const int ks = j % kKStages;
            if (!warp_wait(&bars[B_KEMPTY + ks], ((j / kKStages) & 1) ^ 1, abort_flag, p.d_status)) break;
            uint8_t *kd = sm + kOffK + ks * kTileBytes;
            if (contig) {
                if (leader) {
                    mbar_arrive_expect_tx(&bars[B_KFULL + ks], 2 * kHalfPlane);
                    const int z = PLAIN ? wbase + w : static_cast<int>(b0);
                    tma_load_4d(kd, &tmK8, 0, 0, kvh, z, &bars[B_KFULL + ks]);
                    tma_load_4d(kd + kHalfPlane, &tmK8, kHalfDim, 0, kvh, z, &bars[B_KFULL + ks]);
                }
            } else {
                if (leader) mbar_arrive_expect_tx(&bars[B_KFULL + ks], n * kBlockBytes);
                __syncwarp();
                if (lane < n) {
                    // fully out of bounds: the box is zero-filled
                    const int row = !inb ? p.k_rows
                                         : (PLAIN ? ((wbase + w + lane) * p.hkv + kvh) * kBlockTokens
                                                  : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens);
                    tma_load_2d(kd + lane * kBoxBytes, &tmK, 0, row, &bars[B_KFULL + ks]);
                    tma_load_2d(kd + kHalfPlane + lane * kBoxBytes, &tmK, kHalfDim, row, &bars[B_KFULL + ks]);
                }
            }
            __syncwarp();
            issued = j + 1;
            w += n;
        }
        for (int j = max(0, issued - kKStages); j < issued; ++j)
            mbar_wait(&bars[B_KFULL + j % kKStages], (j / kKStages) & 1);
    } else if (warp == 1) {
        // ============================================================ V producer
        if (leader) tma_prefetch_desc(&tmV);
        int issued = 0;
        for (int w = wbeg, j = 0; w < wend; ++j) {
            const int is = j % kInfoStages;
            if (!warp_wait(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status)) break;
            const int n = info[is].n;
            // lane k < n: block k of the tile
            const uint32_t blk_l = info[is].blk[lane & (kTileBlocks - 1)];
            const uint32_t blk0 = info[is].blk[0];
            bool contig = blk0 < static_cast<uint32_t>(p.num_blocks) &&
                          blk0 + static_cast<uint32_t>(n) <= static_cast<uint32_t>(p.num_blocks);
            contig = __all_sync(0xffffffffu, contig && (lane >= n || blk_l == blk0 + static_cast<uint32_t>(lane)));
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
            const int vs = j % kVStages;
            if (!warp_wait(&bars[B_VEMPTY + vs], ((j / kVStages) & 1) ^ 1, abort_flag, p.d_status)) break;
            uint8_t *vd = sm + kOffV + vs * kTileBytes;
            if (contig) {
                if (leader) {
                    mbar_arrive_expect_tx(&bars[B_VFULL + vs], 2 * kHalfPlane);
                    tma_load_4d(vd, &tmV8, 0, 0, kvh, static_cast<int>(blk0), &bars[B_VFULL + vs]);
                    tma_load_4d(vd + kHalfPlane, &tmV8, kHalfDim, 0, kvh, static_cast<int>(blk0), &bars[B_VFULL + vs]);
                }
            } else {
                if (leader) mbar_arrive_expect_tx(&bars[B_VFULL + vs], n * kBlockBytes);
                __syncwarp();
                if (lane < n) {
                    const int row = blk_l >= static_cast<uint32_t>(p.num_blocks)
                                        ? p.v_rows
                                        : (static_cast<int>(blk_l) * p.hkv + kvh) * kBlockTokens;
                    tma_load_2d(vd + lane * kBoxBytes, &tmV, 0, row, &bars[B_VFULL + vs]);
                    tma_load_2d(vd + kHalfPlane + lane * kBoxBytes, &tmV, kHalfDim, row, &bars[B_VFULL + vs]);
                }
            }
            __syncwarp();
            issued = j + 1;
            w += n;
        }
        for (int j = max(0, issued - kVStages); j < issued; ++j)
            mbar_wait(&bars[B_VFULL + j % kVStages], (j / kVStages) & 1);
    } else if (warp == 2) {
        // ============================================================ MMA issuer
        // One elected lane issues both row tiles' MMAs in the order
        //   QK_0(0) QK_1(0) | PV_0(0) QK_0(1) | PV_1(0) QK_1(1) | PV_0(1) QK_0(2) | ...
        // The tensor core runs them in issue order, so it works on one row tile
        // while the other tile's softmax runs: softmax 0 of tile j+1 overlaps
        // PV_1(j) QK_1(j+1), softmax 1 overlaps PV_0(j+1) QK_0(j+2).  (Two issuers,
        // one per row tile, let the tensor core interleave both tiles' MMAs, which
        // keeps the two softmaxes in step and the tensor core idle while they run.)
        // QK_t(j+1) follows PV_t(j) in issue order, which is what lets P_t live in S_t.
        // The whole warp runs the loop and waits; only the MMAs, commits and
        // arrivals are issued by the elected lane, so the loop state stays uniform.
        const uint32_t idq = tc::idesc_bf16(128, 128, false);
        const uint32_t idv = tc::idesc_bf16(128, 128, true);
        const uint32_t sQ = smem_u32(sm + kOffQ), sK = smem_u32(sm + kOffK), sV = smem_u32(sm + kOffV);
        // descriptors at offset 0 of each buffer; a byte offset b is added as b >> 4
        // to the start-address field (no carry: shared addresses are below 2^18)
        const uint64_t dQ = tc::smem_desc(sQ, 16, 1024), dK0 = tc::smem_desc(sK, 16, 1024);
        const uint64_t dV0 = tc::smem_desc(sV, kHalfPlane, 1024);
        bool ok = warp_wait(&bars[B_QFULL], 0, abort_flag, p.d_status);
        int n = 0, j = 0;
        for (int w = wbeg; ok && w < wend; ++j) {
            // tile j's block count, from the tile-information ring (tile 0's read here,
            // later tiles' one iteration ahead)
            if (j == 0) {
                if (!warp_wait(&bars[B_IFULL], 0, abort_flag, p.d_status)) break;
                n = info[0].n;
                __syncwarp();
                if (leader) mbar_arrive(&bars[B_IEMPTY]);
                if (!warp_wait(ROTK ? &bars[B_KROT] : &bars[B_KFULL], 0, abort_flag, p.d_status)) break;
                tc::fence_after_sync();
                if (leader) {
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t o = static_cast<uint64_t>(((kk >> 2) * kHalfPlane + (kk & 3) * 32) >> 4);
                            tc::mma_ss(tbase + 128 * t, dQ + static_cast<uint64_t>((t * kTileBytes) >> 4) + o, dK0 + o,
                                       idq, kk > 0 ? 1u : 0u);
                        }
                        tc::commit(&bars[B_SFULL + t]);
                    }
                    tc::commit(&bars[B_KEMPTY]);
                }
                __syncwarp();
            }
            const bool next = w + n < wend;
            int n_next = 0;
            const int jn = j + 1, ksn = jn % kKStages;
            if (next) {
                const int is = jn % kInfoStages;
                if (!warp_wait(&bars[B_IFULL + is], (jn / kInfoStages) & 1, abort_flag, p.d_status)) break;
                n_next = info[is].n;
                __syncwarp();
                if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
                // the plain path uses keys as loaded; the lazy path waits for their rotation
                if (!warp_wait(ROTK ? &bars[B_KROT + ksn] : &bars[B_KFULL + ksn], (jn / kKStages) & 1, abort_flag,
                               p.d_status))
                    break;
            }
            const int vs = j % kVStages;
            if (!warp_wait(&bars[B_VFULL + vs], (j / kVStages) & 1, abort_flag, p.d_status)) break;
            const uint64_t vb = dV0 + static_cast<uint64_t>((vs * kTileBytes) >> 4);
            const uint64_t kb = dK0 + static_cast<uint64_t>((ksn * kTileBytes) >> 4);
#pragma unroll 1
            for (int t = 0; t < 2; ++t) {
                if (!warp_wait(&bars[B_PFULL + t], j & 1, abort_flag, p.d_status)) { ok = false; break; }
                tc::fence_after_sync();
                if (leader) {
                    // O_t += P_t V(j); P_t occupies the first 64 columns of S_t
                    for (int k = 0; k < n; ++k)
                        tc::mma_ts(tbase + 256 + 128 * t, tbase + 128 * t + 8 * k,
                                   vb + static_cast<uint64_t>((k * kBoxBytes) >> 4), idv, (j > 0 || k > 0) ? 1u : 0u);
                    tc::commit(&bars[B_ODONE + t]);
                    if (t == 1) tc::commit(&bars[B_VEMPTY + vs]);
                    if (next) {
                        // S_t = Q'_t K(j+1)^T
                        const uint64_t qb = dQ + static_cast<uint64_t>((t * kTileBytes) >> 4);
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint64_t o = static_cast<uint64_t>(((kk >> 2) * kHalfPlane + (kk & 3) * 32) >> 4);
                            tc::mma_ss(tbase + 128 * t, qb + o, kb + o, idq, kk > 0 ? 1u : 0u);
                        }
                        tc::commit(&bars[B_SFULL + t]);
                        if (t == 1) tc::commit(&bars[B_KEMPTY + ksn]);
                    }
                }
                __syncwarp();
            }
            if (!ok) break;
            w += n;
            n = n_next;
        }
        // every MMA this warp issued has completed before tensor memory is freed
        if (leader) tc::commit(&bars[B_DRAIN]);
        __syncwarp();
        mbar_wait(&bars[B_DRAIN], 0);
    } else if (p.q_prep) {
        // ============================================================ prepared query tiles
        // Rows unit * 256 .. + 255 of the prepared query buffer (rotated and scaled by
        // prefill_qprep_kernel): two row tiles, each two 64-column halves of 128 rows.
        if (leader) {
            tma_prefetch_desc(&tmQ);
            mbar_arrive_expect_tx(&bars[B_QFULL], 2 * kTileBytes);
            const int y = unit * kRows;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                tma_load_2d(sm + kOffQ + t * kTileBytes, &tmQ, 0, y + kTileRows * t, &bars[B_QFULL]);
                tma_load_2d(sm + kOffQ + t * kTileBytes + kHalfPlane, &tmQ, kHalfDim, y + kTileRows * t, &bars[B_QFULL]);
            }
        }
        __syncwarp();
        // the loads land before the kernel's tensor memory is freed (the MMAs that read them
        // have completed by then anyway); a wait that runs out only reports
        mbar_wait(&bars[B_QFULL], 0);
    }
    } else if (warp < 12) {
        // ============================================================ softmax (one row per thread)
        // The whole 128-column score row is held in registers: one tensor-memory load
        // and one store (of P) per tile.
        setmaxnreg_inc<kSoftmaxRegs>();
        const int t = (warp - 4) >> 2;                 // row tile
        const int row = threadIdx.x - 128 - 128 * t;   // 0..127 inside the tile
        const int R = R0 + kTileRows * t + row;
        const bool row_ok = R < T * G;
        const int tok = row_ok ? R / G : tok_first;
        const int g = R % G;
        const int prow = pos0 + tok;
        const float slope = ALIBI ? slope_s[g] : 0.f;
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        // Q'_i = R(p_i - P0) q_i for this warpgroup's row tile (R(p_i) on the plain path),
        // unless the tiles arrive prepared by TMA:
        // thread (ch, rb) writes pairs 8ch..8ch+7 of rows rb + 16k; between rows rb + 16k and
        // rb + 16(k+1) the token advances by dlo = 16 / G or dlo + 1, so the angles advance by
        // rotations from two step tables.
        if (!p.q_prep) {
            const int ch = row & 7, rb = row >> 3;
            const int dlo = 16 / G;
            float cA[8], sA[8], cB[8], sB[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                rope_cos_sin(dlo, theta_s[8 * ch + e], cA[e], sA[e]);
                rope_cos_sin(dlo + 1, theta_s[8 * ch + e], cB[e], sB[e]);
            }
            const int qref = PLAIN ? 0 : Pbase;
            {
                const int rowbase = R0 + kTileRows * t + rb;   // global row of k = 0
                int tk_prev = rowbase / G;
                float cc[8], ss[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) rope_cos_sin(pos0 + tk_prev - qref, theta_s[8 * ch + e], cc[e], ss[e]);
                uint8_t *qd = sm + kOffQ + t * kTileBytes;
#pragma unroll 1
                for (int kg = 0; kg < 8; kg += 4) {
                    // issue the global loads of four rows before using any of them
                    uint4 a4[4], b4[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int R = rowbase + 16 * (kg + u);
                        a4[u] = make_uint4(0, 0, 0, 0);
                        b4[u] = make_uint4(0, 0, 0, 0);
                        if (R < T * G) {
                            const uint16_t *q = p.q_raw +
                                                (static_cast<size_t>(q0 + R / G) * p.hq + kvh * G + R % G) * kHeadDim;
                            a4[u] = *reinterpret_cast<const uint4 *>(q + 8 * ch);
                            b4[u] = *reinterpret_cast<const uint4 *>(q + kHalfDim + 8 * ch);
                        }
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int k = kg + u;
                        const int R = rowbase + 16 * k;
                        const int tk = R / G;
                        if (k > 0 && tk != tk_prev) {
                            const bool big = tk - tk_prev != dlo;
#pragma unroll
                            for (int e = 0; e < 8; ++e) {
                                const float sc = big ? cB[e] : cA[e], sn = big ? sB[e] : sA[e];
                                const float c2 = cc[e] * sc - ss[e] * sn;
                                ss[e] = ss[e] * sc + cc[e] * sn;
                                cc[e] = c2;
                            }
                            tk_prev = tk;
                        }
                        const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4[u]);
                        const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4[u]);
                        uint4 lo, hi;
                        uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
                        uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float a0 = bf16_lo(aw[e]) * p.scale_log2, a1 = bf16_hi(aw[e]) * p.scale_log2;
                            const float b0 = bf16_lo(bw[e]) * p.scale_log2, b1 = bf16_hi(bw[e]) * p.scale_log2;
                            const float c0 = cc[2 * e], s0 = ss[2 * e], c1 = cc[2 * e + 1], s1 = ss[2 * e + 1];
                            lw[e] = pack_bf16(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
                            hw[e] = pack_bf16(b0 * c0 + a0 * s0, b1 * c1 + a1 * s1);
                        }
                        const int rw = rb + 16 * k;
                        const uint32_t soff = rw * 128 + ((ch ^ (rw & 7)) << 4);
                        *reinterpret_cast<uint4 *>(qd + soff) = lo;
                        *reinterpret_cast<uint4 *>(qd + kHalfPlane + soff) = hi;
                    }
                }
            }
            fence_proxy_async_smem();   // generic-proxy writes become visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QFULL]);
        }
        const uint32_t tS = tbase + 128 * t, tO = tbase + 256 + 128 * t;
        float m_run = -INFINITY, l_run = 0.f;
        int j = 0;
        bool ok = true;
        for (int w = wbeg; w < wend; ++j) {
            const int is = j % kInfoStages;
            if (!warp_wait(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status)) { ok = false; break; }
            const TileInfo &ti = info[is];
            const int n = ti.n;
            const bool full = (ti.flags & kFull) != 0;
            // visible keys of each 16-key block for this row: slots si < lim_k (0..16), five bits
            // per block in one 64-bit word
            uint64_t limp = 0;
            float bk[kTileBlocks];   // ALiBi: bias of slot 0 of block k, slope * (o + j0 - p); 0 otherwise
#pragma unroll
            for (int k = 0; k < kTileBlocks; ++k) {
                const int nv = k < n ? meta_valid(ti.meta[k]) : 0;
                limp |= static_cast<uint64_t>(max(0, min(nv, prow - ti.off - meta_j0(ti.meta[k]) + 1))) << (5 * k);
                bk[k] = ALIBI ? slope * static_cast<float>(ti.off + meta_j0(ti.meta[k]) - prow) : 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_IEMPTY + is]);
            if (!warp_wait(&bars[B_SFULL + t], j & 1, abort_flag, p.d_status)) { ok = false; break; }
            tc::fence_after_sync();
            // S_t(j) complete implies PV_t(j-1) complete
            uint32_t sv[128];
            tc::ld32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::ld32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            tc::ld32(tS + lane_off + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
            tc::ld32(tS + lane_off + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
            tc::wait_ld();
            if (ALIBI) {
                // the in-block part of the bias, slope * s for slot s; the block part bk[k] enters
                // the block maxima and the exponent's offset below (one op per score, not two)
#pragma unroll
                for (int c = 0; c < 128; c += 2) {
                    float x0 = __uint_as_float(sv[c]), x1 = __uint_as_float(sv[c + 1]);
                    fma2(x0, x1, slope, static_cast<float>(c & 15), static_cast<float>((c + 1) & 15));
                    sv[c] = __float_as_uint(x0);
                    sv[c + 1] = __float_as_uint(x1);
                }
            }
            if (!full) {
#pragma unroll
                for (int k = 0; k < kTileBlocks; ++k) {
                    const int lim = static_cast<int>((limp >> (5 * k)) & 31u);
#pragma unroll
                    for (int c = 16 * k; c < 16 * k + 16; ++c)
                        sv[c] = (c & 15) < lim ? sv[c] : 0xFF800000u;   // -inf: P = 0
                }
            }
            // row max with three-input maxima (exact, so the order does not matter)
            auto f = [&](int c) { return __uint_as_float(sv[c]); };
            float m0 = f(0), m1 = f(1);
            if (ALIBI) {
                // row max of (score + bias): per 16-key block, the block part added once
                m0 = -INFINITY;
#pragma unroll
                for (int k = 0; k < kTileBlocks; ++k) {
                    float a = max3(f(16 * k), f(16 * k + 1), f(16 * k + 2));
#pragma unroll
                    for (int c = 3; c < 15; c += 2) a = max3(a, f(16 * k + c), f(16 * k + c + 1));
                    a = fmaxf(a, f(16 * k + 15));
                    m0 = fmaxf(m0, a + bk[k]);
                }
                m1 = m0;
            } else {
#pragma unroll
                for (int c = 2; c < 126; c += 4) {
                    m0 = max3(m0, f(c), f(c + 1));
                    m1 = max3(m1, f(c + 2), f(c + 3));
                }
                m0 = max3(m0, f(126), f(127));
            }
            const float m_new = fmaxf(m_run, fmaxf(m0, m1));
            const bool need = m_new > m_run + kRescaleThreshold;
            float scale = 1.f;
            if (need) {
                scale = fast_exp2(m_run - m_new);
                m_run = m_new;
                l_run *= scale;
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            // ALiBi: the exponent's offset per block, m - bk[k]
            if (ALIBI) {
#pragma unroll
                for (int k = 0; k < kTileBlocks; ++k) bk[k] = mu - bk[k];
            }
            // P = 2^(S - m) as bf16 pairs over the first 64 columns of S, row sums (even and
            // odd columns) in fp32; the subtraction and the sums run as paired fp32 operations
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const float nmo = -(ALIBI ? bk[e >> 3] : mu);
                float x0 = f(2 * e), x1 = f(2 * e + 1);
                add2(x0, x1, nmo, nmo);
                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                add2(ls0, ls1, p0, p1);
                sv[e] = pack_bf16(p0, p1);
            }
            tc::st32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::st32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            l_run += ls0 + ls1;
            if (j > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::ld32(tO + lane_off + 32 * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
                    tc::st32(tO + lane_off + 32 * c, o);
                }
            }
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_PFULL + t]);
            w += n;
        }
        // ------------------------------------------------------------ epilogue
        bool have = ok && j > 0;
        if (have) have = warp_wait(&bars[B_ODONE + t], (j - 1) & 1, abort_flag, p.d_status);
        const float inv = (have && l_run > 0.f) ? 1.f / l_run : 0.f;
        const bool all_have = __all_sync(0xffffffffu, have);
        if (all_have) tc::fence_after_sync();
        if (part >= 0) {
            // half of a split unit: unnormalised O, running max and sum (log2 domain) for the
            // combine step
            const size_t srow = static_cast<size_t>((unit - p.pf_base) * 2 + part) * kRows + kTileRows * t + row;
            float4 *wo = reinterpret_cast<float4 *>(p.ws_acc + srow * kHeadDim);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t ob[32];
                if (all_have) {
                    tc::ld32(tO + lane_off + 32 * c, ob);
                    tc::wait_ld();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) ob[e] = 0u;
                }
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    wo[8 * c + v] = make_float4(__uint_as_float(ob[4 * v]), __uint_as_float(ob[4 * v + 1]),
                                                __uint_as_float(ob[4 * v + 2]), __uint_as_float(ob[4 * v + 3]));
            }
            p.ws_ml[2 * srow] = have ? m_run : -INFINITY;
            p.ws_ml[2 * srow + 1] = have ? l_run : 0.f;
        }
        uint4 *o = (row_ok && part < 0) ? reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(q0 + tok) * p.hq +
                                                                              kvh * G + g) * kHeadDim)
                                        : nullptr;
#pragma unroll
        for (int c = 0; c < 4 && part < 0; ++c) {
            uint32_t ob[32];
            if (all_have) {
                tc::ld32(tO + lane_off + 32 * c, ob);
                tc::wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) ob[e] = 0u;
            }
            if (o) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 u;
                    u.x = pack_bf16(__uint_as_float(ob[8 * v + 0]) * inv, __uint_as_float(ob[8 * v + 1]) * inv);
                    u.y = pack_bf16(__uint_as_float(ob[8 * v + 2]) * inv, __uint_as_float(ob[8 * v + 3]) * inv);
                    u.z = pack_bf16(__uint_as_float(ob[8 * v + 4]) * inv, __uint_as_float(ob[8 * v + 5]) * inv);
                    u.w = pack_bf16(__uint_as_float(ob[8 * v + 6]) * inv, __uint_as_float(ob[8 * v + 7]) * inv);
                    o[4 * c + v] = u;
                }
            }
        }
    } else {
        // ============================================================ rotations
        setmaxnreg_dec<kRotRegs>();
        // Lazy path only: every K tile, once TMA has landed it, is rotated in
        // shared memory by (o - P0) -- one relative rotation per tile -- so that
        // scores carry the angle (p_i - o - j).  Thread (ch, rb) handles pairs
        // 8ch..8ch+7 of key rows rb + 16k.
        const int tid = threadIdx.x - 384;
        const int ch = tid & 7;
        const int rb = tid >> 3;
        if (ROTK) {
            int cur = INT_MIN;
            float kc[8], kn[8];
            for (int w = wbeg, j = 0; w < wend; ++j) {
                const int is = j % kInfoStages;
                bool okw = wait_or_abort(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status);
                if (!rot_all(okw)) break;
                const int n = info[is].n, off = info[is].off;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_IEMPTY + is]);
                if (off != cur) {
                    cur = off;
#pragma unroll
                    for (int e = 0; e < 8; ++e) rope_cos_sin(off - Pbase, theta_s[8 * ch + e], kc[e], kn[e]);
                }
                const int ks = j % kKStages;
                okw = wait_or_abort(&bars[B_KFULL + ks], (j / kKStages) & 1, abort_flag, p.d_status);
                if (!rot_all(okw)) break;
                uint8_t *kt = sm + kOffK + ks * kTileBytes;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const int row = rb + 16 * k;   // key row of the tile
                    if (row < kBlockTokens * n) {
                        const uint32_t soff = row * 128 + ((ch ^ (row & 7)) << 4);
                        const uint4 a4 = *reinterpret_cast<const uint4 *>(kt + soff);
                        const uint4 b4 = *reinterpret_cast<const uint4 *>(kt + kHalfPlane + soff);
                        const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4);
                        const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4);
                        uint4 lo, hi;
                        uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
                        uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            // (a, b) -> (a c - b s, b c + a s) for two pairs at once (paired fp32)
                            const float a0 = bf16_lo(aw[e]), a1 = bf16_hi(aw[e]);
                            const float b0 = bf16_lo(bw[e]), b1 = bf16_hi(bw[e]);
                            const float c0 = kc[2 * e], s0 = kn[2 * e], c1 = kc[2 * e + 1], s1 = kn[2 * e + 1];
                            float ac0, ac1, bc0, bc1, lo0, lo1, hi0, hi1;
                            mul2(ac0, ac1, a0, a1, c0, c1);
                            mul2(bc0, bc1, b0, b1, c0, c1);
                            fma2v(lo0, lo1, -b0, -b1, s0, s1, ac0, ac1);
                            fma2v(hi0, hi1, a0, a1, s0, s1, bc0, bc1);
                            lw[e] = pack_bf16(lo0, lo1);
                            hw[e] = pack_bf16(hi0, hi1);
                        }
                        *reinterpret_cast<uint4 *>(kt + soff) = lo;
                        *reinterpret_cast<uint4 *>(kt + kHalfPlane + soff) = hi;
                    }
                }
                fence_proxy_async_smem();   // the tensor core reads the rotated tile
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_KROT + ks]);
                w += n;
            }
        }
    }

    // ================================================================ teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 2) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, 512);
    }
}

// Merges the two halves of each split unit: with M = max(m0, m1) and w_i = 2^(m_i - M),
// O = (w0 O0 + w1 O1) / (w0 l0 + w1 l1) -- the same merge as between consecutive key tiles
// of one CTA.  One warp per query row, 4 columns of d per lane.
__global__ void __launch_bounds__(256) prefill_combine_kernel(const AttnParams p) {
    const int s = blockIdx.x, row_in = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int unit = p.pf_base + s;
    const int mt = unit % p.pf_mtiles, kvh = (unit / p.pf_mtiles) % p.hkv, r = unit / (p.pf_mtiles * p.hkv);
    const int G = p.group;
    const int q0 = p.cu_q[r], T = p.cu_q[r + 1] - q0;
    const int R = mt * kRows + row_in;
    if (R >= T * G) return;
    const size_t r0 = static_cast<size_t>(2 * s) * kRows + row_in, r1 = r0 + kRows;
    const float m0 = p.ws_ml[2 * r0], l0 = p.ws_ml[2 * r0 + 1], m1 = p.ws_ml[2 * r1], l1 = p.ws_ml[2 * r1 + 1];
    const float M = fmaxf(m0, m1);
    const float w0 = m0 == -INFINITY ? 0.f : exp2f(m0 - M), w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - M);
    const float L = w0 * l0 + w1 * l1;
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const float4 a = reinterpret_cast<const float4 *>(p.ws_acc + r0 * kHeadDim)[lane];
    const float4 b = reinterpret_cast<const float4 *>(p.ws_acc + r1 * kHeadDim)[lane];
    uint2 u;
    u.x = pack_bf16((w0 * a.x + w1 * b.x) * inv, (w0 * a.y + w1 * b.y) * inv);
    u.y = pack_bf16((w0 * a.z + w1 * b.z) * inv, (w0 * a.w + w1 * b.w) * inv);
    const int tok = R / G, g = R % G;
    reinterpret_cast<uint2 *>(p.out + (static_cast<size_t>(q0 + tok) * p.hq + kvh * G + g) * kHeadDim)[lane] = u;
}

// The query tiles of every work unit, rotated and scaled, ahead of the attention kernel:
// row R of unit (m-tile mt, KV head kvh, request r) -- token R / G, head kvh * G + R % G --
// becomes Q'_R = scale_log2 * R(p - qref) q at buffer row unit * 256 + R % 256, with
// qref = P0 = q_pos0[r] + (256 mt) / G, the unit's first query position (0 on the plain path:
// rotation to the absolute position).  Rows past the request's tokens are zero.  One thread
// per (request, row, group of 8 rotation pairs); the angles of its 8 pairs are evaluated once
// and applied to the row of every KV head.
__global__ void __launch_bounds__(256) prefill_qprep_kernel(const AttnParams p, int plain) {
    const int r = blockIdx.y;
    const int R = blockIdx.x * 32 + (threadIdx.x >> 3), ch = threadIdx.x & 7;
    const int G = p.group;
    const int q0 = p.cu_q[r], T = p.cu_q[r + 1] - q0;
    const int mt = R / kRows;
    if (mt >= p.pf_mtiles || mt * kRows >= T * G) return;   // no unit of this request holds row R
    const size_t dst_row0 = (static_cast<size_t>(r) * p.hkv * p.pf_mtiles + mt) * kRows + R % kRows;
    const size_t unit_stride = static_cast<size_t>(p.pf_mtiles) * kRows;   // next KV head, same m-tile
    if (R >= T * G) {
        for (int kvh = 0; kvh < p.hkv; ++kvh) {
            uint4 *d = reinterpret_cast<uint4 *>(p.q_prep + (dst_row0 + kvh * unit_stride) * kHeadDim);
            d[ch] = make_uint4(0, 0, 0, 0);
            d[8 + ch] = make_uint4(0, 0, 0, 0);
        }
        return;
    }
    const int tok = R / G, g = R % G;
    const int pos0 = p.q_pos0[r];
    const int delta = plain ? pos0 + tok : tok - (mt * kRows) / G;
    float c[8], sn[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) rope_cos_sin(delta, p.rope.theta[8 * ch + e], c[e], sn[e]);
    const float sc = p.scale_log2;
    // eight KV heads at a time: all loads issued before the first store
    constexpr int kHeadsPerPass = 8;
    for (int kb = 0; kb < p.hkv; kb += kHeadsPerPass) {
        uint4 a8[kHeadsPerPass], b8[kHeadsPerPass];
#pragma unroll
        for (int u = 0; u < kHeadsPerPass; ++u) {
            if (kb + u < p.hkv) {
                const uint4 *q = reinterpret_cast<const uint4 *>(
                    p.q_raw + (static_cast<size_t>(q0 + tok) * p.hq + (kb + u) * G + g) * kHeadDim);
                a8[u] = __ldg(q + ch);
                b8[u] = __ldg(q + 8 + ch);
            }
        }
#pragma unroll
        for (int u = 0; u < kHeadsPerPass; ++u) {
            if (kb + u >= p.hkv) break;
            const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a8[u]);
            const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b8[u]);
            uint4 lo, hi;
            uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
            uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float a0 = bf16_lo(aw[e]) * sc, a1 = bf16_hi(aw[e]) * sc;
                const float b0 = bf16_lo(bw[e]) * sc, b1 = bf16_hi(bw[e]) * sc;
                const float c0 = c[2 * e], s0 = sn[2 * e], c1 = c[2 * e + 1], s1 = sn[2 * e + 1];
                lw[e] = pack_bf16(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
                hw[e] = pack_bf16(b0 * c0 + a0 * s0, b1 * c1 + a1 * s1);
            }
            uint4 *d = reinterpret_cast<uint4 *>(p.q_prep + (dst_row0 + (kb + u) * unit_stride) * kHeadDim);
            d[ch] = lo;
            d[8 + ch] = hi;
        }
    }
}

template <int MODE>
cudaError_t launch_t(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8, const CUtensorMap &tv8,
                     const CUtensorMap &tq, const AttnParams &p, cudaStream_t s) {
    auto kern = prefill_tc_kernel<MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmem);
    if (e != cudaSuccess) return e;
    static_assert(kRows == kPrefillRows, "rows per CTA");
    if (p.q_prep) {
        prefill_qprep_kernel<<<dim3(p.pf_mtiles * (kRows / 32), p.num_req), 256, 0, s>>>(p, MODE == kPlain);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    kern<<<p.pf_base + 2 * p.pf_nsplit, kThreads, kTcSmem, s>>>(tk, tv, tk8, tv8, tq, p);
    e = cudaGetLastError();
    if (e != cudaSuccess || p.pf_nsplit == 0) return e;
    prefill_combine_kernel<<<dim3(p.pf_nsplit, kRows / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                              const CUtensorMap &tv8, const CUtensorMap &tq, const AttnParams &p, bool plain,
                              cudaStream_t s) {
    if (plain) return launch_t<kPlain>(tk, tv, tk8, tv8, tq, p, s);
    return p.alibi ? launch_t<kAlibi>(tk, tv, tk8, tv8, tq, p, s) : launch_t<kLazy>(tk, tv, tk8, tv8, tq, p, s);
}

}  // namespace lazy
