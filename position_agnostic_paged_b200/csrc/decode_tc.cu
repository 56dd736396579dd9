// decode_tc.cu -- decode attention for many query heads per KV head (G > 8, MQA
// included) on the fifth-generation tensor cores.
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Decoding -- one query token per request; the query is
// rotated again only when the segment offset changes (a new document); the
// keys are used as the pool stores them (rotated at their local index j), so
// the kernel reads only K and V.
//
// Why tensor memory here.  With G heads sharing one KV head, every 16-key
// block feeds G x 16 scores: for G = 32 the contraction per K/V byte is 32
// FLOP/B, which warp-level MMAs with the heads as 16-row tiles could not keep
// up with at HBM speed (their accumulators cap the CTAs per SM).  Here the
// heads are the rows of 128 x 128 tcgen05 MMAs (rows G..127 are padding whose
// results are never read), scores and the output accumulate in tensor memory,
// and one CTA per SM streams 128-key tiles through three-stage K and V rings.
//
// CTA = one split (a range of table words) of one KV head of one request.
// Tiles are up to 8 consecutive words of one segment.  Two softmax streams
// take alternate tiles (stream t = tile index mod 2), each with its own score
// buffer S_t, output accumulator O_t and online-softmax state, so that one
// stream's softmax overlaps the other stream's MMAs; each stream writes its
// own split partial and the combine kernel merges them with the other splits.
//   warp 0   K producer: walks the table one word per lane, publishes tile
//            information, TMA-loads each tile's K into a ring of three stages
//   warp 3   V producer (and owner of tensor memory): each tile's V into a ring
//            of its own, so that a V stage held until PV does not hold back K
//   warp 1   MMA issuer: QK(j) into S_{j%2} and PV(j-1) from P_{(j-1)%2}, in the
//            order their inputs become ready
//   warp 2   query rotation: Q' = R(q_pos - o) q * scale for each new segment
//            offset o, computed ahead and stored into the single query buffer
//            once the previous one is no longer read; the G heads are written
//            twice, as rows 0..G-1 and 32..32+G-1
//   warp 4   softmax of stream 0: tensor-memory lanes 0-31 (rows 0-31)
//   warp 5   softmax of stream 1: lanes 32-63 (rows 32-63, the second copy of
//            the heads), so that the two streams' softmaxes run on different
//            sub-partitions of the SM
//   warps 6-7 copy the 64 rotation frequencies to shared memory at the start
// Tensor memory (512 columns): S0 [0,128) (P0 = its first 64 columns),
// S1 [128,256) (P1), O0 [256,384), O1 [384,512).
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lazy {

namespace {

constexpr int kTB = 8;                              // blocks per tile
constexpr int kTileB = 128 * kHeadDim * 2;          // 32 KiB: 128 rows of 128 bf16
constexpr int kHalfP = kTileB / 2;                  // 16 KiB: one 64-column half plane
constexpr int kStages = 3, kInfo = 8;
constexpr int kThreadsTc = 256;                     // 8 warps

struct DInfo {
    uint32_t blk[kTB];
    uint32_t meta[kTB];
    int n;       // blocks in the tile (1..8)
    int off;     // the segment's logical offset
    int flags;   // kAllVisible: every key of the tile is visible to the query
    int pad;
};
constexpr int kAllVisible = 1;
static_assert(sizeof(DInfo) == 80, "tile info layout");

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kTileB;
constexpr int kOffV = kOffK + kStages * kTileB;
constexpr int kOffInfo = kOffV + kStages * kTileB;
constexpr int kOffBar = kOffInfo + kInfo * static_cast<int>(sizeof(DInfo));
constexpr int B_KFULL = 0, B_KEMPTY = B_KFULL + kStages, B_VFULL = B_KEMPTY + kStages,
              B_VEMPTY = B_VFULL + kStages, B_IFULL = B_VEMPTY + kStages,
              B_IEMPTY = B_IFULL + kInfo, B_SFULL = B_IEMPTY + kInfo, B_PFULL = B_SFULL + 2,
              B_ODONE = B_PFULL + 2, B_QREADY = B_ODONE + 2, B_QFREE = B_QREADY + 1, B_DRAIN = B_QFREE + 1,
              kBars = B_DRAIN + 1;
constexpr int kOffCs = kOffBar + kBars * 8;         // cos, sin of the 64 rotation angles (float2)
constexpr int kOffMisc = kOffCs + kHalfDim * 8;     // tensor-memory address, abort flag
constexpr int kOffTheta = kOffMisc + 16;            // the 64 rotation frequencies (double)
constexpr int kSmemUse = kOffTheta + kHalfDim * 8;
constexpr size_t kSmemTc = kSmemUse + 1024;
static_assert(kSmemTc <= 232448, "shared memory budget");
// consumers of a tile-information entry: the V producer, the issuer, the rotation warp, both
// softmax warps
constexpr int kInfoReaders = 5;
constexpr float kRescale = 8.0f;   // log2 units: P stays below 2^8 between rescales

__device__ __forceinline__ uint8_t *align1k(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ void tma4d(void *dst, const CUtensorMap *map, int x, int y, int h, int b, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(h), "r"(b), "r"(smem_u32(bar))
        : "memory");
}
// Same decision for every lane of the warp.
__device__ __forceinline__ bool wwait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *d_status) {
    const bool ok = wait_or_abort(bar, parity, abort_flag, d_status);
    return __all_sync(0xffffffffu, ok);
}

// MODE: 0 lazy (pool keys, query rotated by q_pos - o per segment), 1 plain (keys materialised
// at absolute positions, indexed by table position; query rotated once by q_pos), 2 ALiBi
// (nothing rotated, bias slope_h * (key position - q_pos) added to each score).
template <int MODE>
// one CTA per SM (shared memory allows no more)
__global__ void __launch_bounds__(kThreadsTc, 1) decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                  const __grid_constant__ CUtensorMap tmV,
                                                  const __grid_constant__ CUtensorMap tmK8,
                                                  const __grid_constant__ CUtensorMap tmV8, const AttnParams p) {
    constexpr bool PLAIN = MODE == 1;
    constexpr bool ALIBI = MODE == 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1k(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    DInfo *info = reinterpret_cast<DInfo *>(sm + kOffInfo);
    float2 *cs = reinterpret_cast<float2 *>(sm + kOffCs);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    double *theta_s = reinterpret_cast<double *>(sm + kOffTheta);

    const int split = blockIdx.x, kvh = blockIdx.y, r = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    const int lo = split * p.words_per_split;
    const int hi = max(lo, min(n_words, lo + p.words_per_split));
    const uint32_t *tbl = p.table + wbase;
    const int qpos = p.q_pos[r];

    // The K producer's first table words, loaded before the barrier set-up; the two idle warps
    // copy the rotation frequencies to shared memory meanwhile (per-lane reads of the parameter
    // table serialise, so the rotation warp does not make them).
    uint32_t first_wl = 0xFFFFFFFFu;
    if (warp == 0 && lane < kTB && lo + lane < hi) first_wl = tbl[lo + lane];
    if (warp >= 6) theta_s[32 * (warp - 6) + lane] = p.rope.theta[32 * (warp - 6) + lane];

    if (threadIdx.x == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], 1);
            mbar_init(&bars[B_VFULL + i], 1);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        for (int i = 0; i < kInfo; ++i) {
            mbar_init(&bars[B_IFULL + i], 1);
            mbar_init(&bars[B_IEMPTY + i], kInfoReaders);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&bars[B_SFULL + t], 1);
            mbar_init(&bars[B_PFULL + t], 1);
            mbar_init(&bars[B_ODONE + t], 1);
        }
        mbar_init(&bars[B_QREADY], 1);
        mbar_init(&bars[B_QFREE], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        if (split == 0 && kvh == 0 && n_words > p.max_words) set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (warp == 3) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const bool leader = tc::elect_one();

    if (warp == 0) {
        // ============================================================ table walk + K/V producer
        if (leader) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
        }
        int issued = 0;
        for (int w = lo, j = 0; w < hi; ++j) {
            // the tile: up to 8 consecutive words sharing one offset; lane k < 8 holds word k
            const uint32_t wl = j == 0 ? first_wl : ((lane < kTB && w + lane < hi) ? tbl[w + lane] : 0xFFFFFFFFu);
            const int off = word_offset(__shfl_sync(0xffffffffu, wl, 0));
            const bool same = lane < kTB && w + lane < hi && word_offset(wl) == off;
            const int n = __ffs(~__ballot_sync(0xffffffffu, same)) - 1;   // lanes 0..n-1 share it
            const uint32_t b = word_block(wl);
            const bool inb = lane < n && b < static_cast<uint32_t>(p.num_blocks);
            const uint32_t mt = inb ? p.blk_meta[b] : 0u;   // a bad block has no valid slot
            if (lane < n && !inb) set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
            const bool all_vis =
                n == kTB && __all_sync(0xffffffffu, lane >= n || (meta_valid(mt) == kBlockTokens &&
                                                                   off + meta_j0(mt) + kBlockTokens - 1 <= qpos));
            const uint32_t b0 = __shfl_sync(0xffffffffu, b, 0);
            // blocks consecutive in the pool: two 16 KiB boxes per operand instead of 2n small ones
            const bool contig = __all_sync(0xffffffffu, lane >= n || (inb && b == b0 + static_cast<uint32_t>(lane)));
            const int is = j % kInfo;
            if (!wwait(&bars[B_IEMPTY + is], ((j / kInfo) & 1) ^ 1, abort_flag, p.d_status)) break;
            DInfo &ti = info[is];
            if (lane < kTB) {
                ti.blk[lane] = lane < n ? b : 0u;
                ti.meta[lane] = mt;
            }
            if (leader) {
                ti.n = n;
                ti.off = off;
                ti.flags = all_vis ? kAllVisible : 0;
            }
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_IFULL + is]);
            // K tile; its stage is free again once QK of the tile three back has completed
            const int st = j % kStages;
            if (!wwait(&bars[B_KEMPTY + st], ((j / kStages) & 1) ^ 1, abort_flag, p.d_status)) break;
            uint8_t *kd = sm + kOffK + st * kTileB;
            uint64_t *fb = &bars[B_KFULL + st];
            const bool k_contig = PLAIN || contig;   // the materialised copy is indexed by table position
            if (leader) {
                mbar_arrive_expect_tx(fb, k_contig ? 2 * kHalfP : n * kBlockBytes);
                if (k_contig) {
                    const int z = PLAIN ? wbase + w : static_cast<int>(b0);
                    tma4d(kd, &tmK8, 0, 0, kvh, z, fb);
                    tma4d(kd + kHalfP, &tmK8, kHalfDim, 0, kvh, z, fb);
                }
            }
            __syncwarp();
            if (!k_contig && lane < n) {
                // fully out of bounds: the box is zero-filled
                const int row = !inb ? p.k_rows : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                tma_load_2d(kd + lane * kBoxBytes, &tmK, 0, row, fb);
                tma_load_2d(kd + kHalfP + lane * kBoxBytes, &tmK, kHalfDim, row, fb);
            }
            __syncwarp();
            issued = j + 1;
            w += n;
        }
        // every copy has landed before the kernel ends
        for (int j = max(0, issued - kStages); j < issued; ++j)
            mbar_wait(&bars[B_KFULL + j % kStages], (j / kStages) & 1);
    } else if (warp == 3) {
        // ============================================================ V producer
        // V tiles in their own ring: a V stage is held from its load until PV of its tile, so
        // loading it in step with K would tie the K loads to the much later PV.
        if (leader) tma_prefetch_desc(&tmV);
        int issued = 0;
        for (int w = lo, j = 0; w < hi; ++j) {
            const int is = j % kInfo;
            if (!wwait(&bars[B_IFULL + is], (j / kInfo) & 1, abort_flag, p.d_status)) break;
            const int n = info[is].n;
            const uint32_t blk_l = info[is].blk[lane & (kTB - 1)];   // lane b < n: block b of the tile
            const uint32_t blk0 = info[is].blk[0];
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
            const bool inb = lane < n && blk_l < static_cast<uint32_t>(p.num_blocks);
            const bool contig =
                __all_sync(0xffffffffu, lane >= n || (inb && blk_l == blk0 + static_cast<uint32_t>(lane)));
            const int st = j % kStages;
            if (!wwait(&bars[B_VEMPTY + st], ((j / kStages) & 1) ^ 1, abort_flag, p.d_status)) break;
            uint8_t *vd = sm + kOffV + st * kTileB;
            uint64_t *fb = &bars[B_VFULL + st];
            if (leader) {
                mbar_arrive_expect_tx(fb, contig ? 2 * kHalfP : n * kBlockBytes);
                if (contig) {
                    tma4d(vd, &tmV8, 0, 0, kvh, static_cast<int>(blk0), fb);
                    tma4d(vd + kHalfP, &tmV8, kHalfDim, 0, kvh, static_cast<int>(blk0), fb);
                }
            }
            __syncwarp();
            if (!contig && lane < n) {
                const int row = !inb ? p.v_rows : (static_cast<int>(blk_l) * p.hkv + kvh) * kBlockTokens;
                tma_load_2d(vd + lane * kBoxBytes, &tmV, 0, row, fb);
                tma_load_2d(vd + kHalfP + lane * kBoxBytes, &tmV, kHalfDim, row, fb);
            }
            __syncwarp();
            issued = j + 1;
            w += n;
        }
        for (int j = max(0, issued - kStages); j < issued; ++j)
            mbar_wait(&bars[B_VFULL + j % kStages], (j / kStages) & 1);
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        // Order QK(0) | QK(1) PV(0) | QK(2) PV(1) | ...: S_t(j) (t = j % 2) is computed while the
        // other stream's softmax runs, and QK(j) follows PV(j-2) in issue order, which is what lets
        // P_t live in S_t.  A new segment offset needs a new query: QFREE is committed after the
        // last MMA that reads the old one, and the rotation warp publishes the new one (QREADY).
        const uint32_t idq = tc::idesc_bf16(128, 128, false);
        const uint32_t idv = tc::idesc_bf16(128, 128, true);
        const uint64_t dQ = tc::smem_desc(smem_u32(sm + kOffQ), 16, 1024);
        const uint64_t dK0 = tc::smem_desc(smem_u32(sm + kOffK), 16, 1024);
        const uint64_t dV0 = tc::smem_desc(smem_u32(sm + kOffV), kHalfP, 1024);
        // Two actions are pending at a time: QK(j) (needs K/V tile j and, at a new offset, the new
        // query) and PV(j-1) (needs P(j-1)); whichever is ready first is issued, QK(j) first when
        // both are, so that neither waits behind the other's producer.
        int prev_n = 0, gen = -1, cur_rot = INT_MIN, j = 0;
        bool ok = true, prev_tile = false;   // prev_tile: tile j-1 exists (and still needs its PV)
        for (int w = lo; ok; ++j) {
            const bool has_qk = w < hi;
            int n = 0;
            if (has_qk) {
                const int is = j % kInfo;
                if (!wwait(&bars[B_IFULL + is], (j / kInfo) & 1, abort_flag, p.d_status)) { ok = false; break; }
                n = info[is].n;
                const int off = info[is].off;
                __syncwarp();
                if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
                const int rot = PLAIN ? 0 : (ALIBI ? qpos : off);
                if (rot != cur_rot) {
                    // every MMA that read the previous query has been issued (QK(j-1) at the latest)
                    cur_rot = rot;
                    ++gen;
                    if (gen > 0 && leader) tc::commit(&bars[B_QFREE]);
                    __syncwarp();
                }
            }
            const bool has_pv = prev_tile;
            if (!has_qk && !has_pv) break;
            bool need_qk = has_qk, need_pv = has_pv, need_q = has_qk;   // need_q: query not yet seen ready
            const int st = j % kStages, t = j & 1;
            const int u = (j - 1) & 1, su = (j + kStages - 1) % kStages;
            uint32_t polls = 0;
            while (need_qk || need_pv) {
                if (need_qk) {
                    if (need_q) need_q = !__all_sync(0xffffffffu, mbar_test_wait(&bars[B_QREADY], gen & 1));
                    if (!need_q && __all_sync(0xffffffffu, mbar_test_wait(&bars[B_KFULL + st], (j / kStages) & 1))) {
                        tc::fence_after_sync();
                        if (leader) {
                            const uint64_t kb = dK0 + static_cast<uint64_t>((st * kTileB) >> 4);
#pragma unroll
                            for (int kk = 0; kk < 8; ++kk) {
                                const uint64_t o = static_cast<uint64_t>(((kk >> 2) * kHalfP + (kk & 3) * 32) >> 4);
                                tc::mma_ss(tbase + 128 * t, dQ + o, kb + o, idq, kk > 0 ? 1u : 0u);
                            }
                            tc::commit(&bars[B_SFULL + t]);
                            tc::commit(&bars[B_KEMPTY + st]);
                        }
                        __syncwarp();
                        need_qk = false;
                        continue;
                    }
                }
                if (need_pv && __all_sync(0xffffffffu, mbar_test_wait(&bars[B_PFULL + u], ((j - 1) >> 1) & 1) &&
                                                           mbar_test_wait(&bars[B_VFULL + su], ((j - 1) / kStages) & 1))) {
                    // PV(j-1): O_u += P_u V(j-1), P_u in the first 64 columns of S_u
                    tc::fence_after_sync();
                    if (leader) {
                        const uint64_t vb = dV0 + static_cast<uint64_t>((su * kTileB) >> 4);
                        for (int k = 0; k < prev_n; ++k)
                            tc::mma_ts(tbase + 256 + 128 * u, tbase + 128 * u + 8 * k,
                                       vb + static_cast<uint64_t>((k * kBoxBytes) >> 4), idv,
                                       (j - 1 > 1 || k > 0) ? 1u : 0u);
                        tc::commit(&bars[B_ODONE + u]);
                        tc::commit(&bars[B_VEMPTY + su]);
                    }
                    __syncwarp();
                    need_pv = false;
                    continue;
                }
                // nothing ready: bounded, like every other wait
                if (++polls > (kWaitPolls << 2) || ((polls & 255) == 0 && *abort_flag)) {
                    if (polls > (kWaitPolls << 2)) {
                        *abort_flag = 1;
                        if (leader) set_status(p.d_status, LAZY_DSTATUS_TIMEOUT);
                    }
                    ok = false;
                    break;
                }
            }
            prev_n = n;
            prev_tile = has_qk;
            w += n;
        }
        // every MMA this warp issued has completed before tensor memory is freed
        if (leader) tc::commit(&bars[B_DRAIN]);
        __syncwarp();
        mbar_wait(&bars[B_DRAIN], 0);
    } else if (warp == 2) {
        // ============================================================ query rotation
        // Q'_h = R(q_pos - o) q_h * scale_log2 for each new offset o (once, by q_pos, on the plain
        // path; the identity under ALiBi), lane h writing head h's row of the MMA A operand
        // (K-major, 128-byte swizzle, two 64-column half planes).  The angles are evaluated once
        // per rotation, two per lane (frequencies from shared memory), and shared through shared
        // memory.  The raw query row is
        // loaded once and kept in registers, and the first query is made from the first table
        // word, read here, before the tile information is published (the issuer sees the same
        // offset in the first entry): it is ready about when the first K tile lands.
        uint4 qa[8], qb[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            qa[c] = make_uint4(0, 0, 0, 0);
            qb[c] = make_uint4(0, 0, 0, 0);
        }
        int first_rot = PLAIN ? 0 : qpos;
        if (lo < hi) {
            if (lane < G) {
                const uint4 *qrow = reinterpret_cast<const uint4 *>(
                    p.q_raw + (static_cast<size_t>(r) * p.hq + kvh * G + lane) * kHeadDim);
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    qa[c] = __ldg(qrow + c);       // elements 8c .. 8c + 7
                    qb[c] = __ldg(qrow + 8 + c);   // elements 64 + 8c ..
                }
            }
            if (!PLAIN && !ALIBI) first_rot = word_offset(tbl[lo]);
        }
        int gen = -1, cur_rot = INT_MIN;
        const float sc = p.scale_log2;
        bool first = true;
        for (int w = lo, j = 0; w < hi;) {
            int rot = first_rot;
            if (!first) {
                const int is = j % kInfo;
                if (!wwait(&bars[B_IFULL + is], (j / kInfo) & 1, abort_flag, p.d_status)) break;
                const int n = info[is].n, off = info[is].off;
                __syncwarp();
                if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
                w += n;
                ++j;
                rot = PLAIN ? 0 : (ALIBI ? qpos : off);
            }
            first = false;
            if (rot == cur_rot) continue;
            cur_rot = rot;
            ++gen;
            // The new query is computed into registers as soon as its offset is known; only the
            // store waits until the previous query is no longer read (every MMA issued before
            // QFREE completed).
            const int delta = qpos - rot;
            float c0, s0, c1, s1;
            rope_cos_sin(delta, theta_s[lane], c0, s0);
            rope_cos_sin(delta, theta_s[lane + 32], c1, s1);
            __syncwarp();   // the previous rotation's reads of the angle table are done
            cs[lane] = make_float2(c0, s0);
            cs[lane + 32] = make_float2(c1, s1);
            __syncwarp();
            uint4 lo8[8], hi8[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                lo8[c] = make_uint4(0, 0, 0, 0);
                hi8[c] = make_uint4(0, 0, 0, 0);
            }
            if (lane < G) {
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    // keeps the unpacked, scaled query from being hoisted out of the loop (128
                    // floats held across it would not fit the registers)
                    asm volatile("" : "+r"(qa[c].x), "+r"(qa[c].y), "+r"(qa[c].z), "+r"(qa[c].w));
                    asm volatile("" : "+r"(qb[c].x), "+r"(qb[c].y), "+r"(qb[c].z), "+r"(qb[c].w));
                }
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const uint32_t *aw = reinterpret_cast<const uint32_t *>(&qa[c]);
                    const uint32_t *bw = reinterpret_cast<const uint32_t *>(&qb[c]);
                    uint32_t *lw = reinterpret_cast<uint32_t *>(&lo8[c]);
                    uint32_t *hw = reinterpret_cast<uint32_t *>(&hi8[c]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 q0 = cs[8 * c + 2 * e], q1 = cs[8 * c + 2 * e + 1];
                        const float a0 = bf16_lo(aw[e]) * sc, a1 = bf16_hi(aw[e]) * sc;
                        const float b0 = bf16_lo(bw[e]) * sc, b1 = bf16_hi(bw[e]) * sc;
                        lw[e] = pack_bf16(a0 * q0.x - b0 * q0.y, a1 * q1.x - b1 * q1.y);
                        hw[e] = pack_bf16(b0 * q0.x + a0 * q0.y, b1 * q1.x + a1 * q1.y);
                    }
                }
            }
            if (gen > 0 && !wwait(&bars[B_QFREE], (gen - 1) & 1, abort_flag, p.d_status)) break;
            uint8_t *qd = sm + kOffQ;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                // rows lane and 32 + lane (same swizzle phase: 32 is a multiple of 8)
                const uint32_t soff = lane * 128 + ((c ^ (lane & 7)) << 4);
                *reinterpret_cast<uint4 *>(qd + soff) = lo8[c];
                *reinterpret_cast<uint4 *>(qd + kHalfP + soff) = hi8[c];
                *reinterpret_cast<uint4 *>(qd + 32 * 128 + soff) = lo8[c];
                *reinterpret_cast<uint4 *>(qd + kHalfP + 32 * 128 + soff) = hi8[c];
            }
            fence_proxy_async_smem();   // generic-proxy writes become visible to the tensor core
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_QREADY]);
        }
    } else if (warp == 4 || warp == 5) {
        // ============================================================ softmax (one head per lane)
        // Stream t takes tiles j with j % 2 == t; every tile's information is read (to follow the
        // word ranges), only the stream's own tiles are processed.  The whole 128-column score
        // row of the lane's head is held in registers: one tensor-memory load, mask, max,
        // 2^(S - m), one store of P over the consumed S columns; O rescaled lazily.
        const int t = warp - 4;
        // stream t's rows 32t .. 32t + 31 = tensor-memory lanes of this warp's quarter
        const uint32_t lane_off = static_cast<uint32_t>(32 * t) << 16;
        const uint32_t tS = tbase + lane_off + 128 * t, tO = tbase + lane_off + 256 + 128 * t;
        const float slope = (ALIBI && lane < G) ? p.alibi_log2[kvh * G + lane] : 0.f;
        float m_run = -INFINITY, l_run = 0.f;
        int k = 0;   // tiles of this stream processed
        bool ok = true;
        for (int w = lo, j = 0; w < hi; ++j) {
            const int is = j % kInfo;
            if (!wwait(&bars[B_IFULL + is], (j / kInfo) & 1, abort_flag, p.d_status)) { ok = false; break; }
            const DInfo &ti = info[is];
            const int n = ti.n, off = ti.off;
            const bool all_vis = (ti.flags & kAllVisible) != 0;
            // visible slots of each block: si < lim_b (0..16), five bits per block
            uint64_t limp = 0;
            float bk[kTB];   // ALiBi: bias of slot 0 of block b, slope * (o + j0 - q_pos)
#pragma unroll
            for (int b = 0; b < kTB; ++b) {
                const uint32_t mb = ti.meta[b];
                const int nv = b < n ? meta_valid(mb) : 0;
                limp |= static_cast<uint64_t>(max(0, min(nv, qpos - off - meta_j0(mb) + 1))) << (5 * b);
                bk[b] = ALIBI ? slope * static_cast<float>(off + meta_j0(mb) - qpos) : 0.f;
            }
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_IEMPTY + is]);
            w += n;
            if ((j & 1) != t) continue;
            if (!wwait(&bars[B_SFULL + t], k & 1, abort_flag, p.d_status)) { ok = false; break; }
            tc::fence_after_sync();
            // S_t(j) complete implies PV_t(j-2) complete: O_t is settled and P_t(j-2) was read
            uint32_t sv[128];
            tc::ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            tc::ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
            tc::ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
            tc::wait_ld();
            if (ALIBI) {
                // the in-block part of the bias, slope * s for slot s
#pragma unroll
                for (int c = 0; c < 128; c += 2) {
                    float x0 = __uint_as_float(sv[c]), x1 = __uint_as_float(sv[c + 1]);
                    fma2(x0, x1, slope, static_cast<float>(c & 15), static_cast<float>((c + 1) & 15));
                    sv[c] = __float_as_uint(x0);
                    sv[c + 1] = __float_as_uint(x1);
                }
            }
            if (!all_vis) {
#pragma unroll
                for (int b = 0; b < kTB; ++b) {
                    const int lim = static_cast<int>((limp >> (5 * b)) & 31u);
#pragma unroll
                    for (int c = 16 * b; c < 16 * b + 16; ++c)
                        sv[c] = (c & 15) < lim ? sv[c] : 0xFF800000u;   // -inf: P = 0
                }
            }
            auto f = [&](int c) { return __uint_as_float(sv[c]); };
            float m0, m1;
            if (ALIBI) {
                m0 = -INFINITY;
#pragma unroll
                for (int b = 0; b < kTB; ++b) {
                    float a = max3(f(16 * b), f(16 * b + 1), f(16 * b + 2));
#pragma unroll
                    for (int c = 3; c < 15; c += 2) a = max3(a, f(16 * b + c), f(16 * b + c + 1));
                    a = fmaxf(a, f(16 * b + 15));
                    m0 = fmaxf(m0, a + bk[b]);
                }
                m1 = m0;
            } else {
                m0 = f(0);
                m1 = f(1);
#pragma unroll
                for (int c = 2; c < 126; c += 4) {
                    m0 = max3(m0, f(c), f(c + 1));
                    m1 = max3(m1, f(c + 2), f(c + 3));
                }
                m0 = max3(m0, f(126), f(127));
            }
            const float m_new = fmaxf(m_run, fmaxf(m0, m1));
            const bool need = m_new > m_run + kRescale;
            float scale = 1.f;
            if (need) {
                scale = fast_exp2(m_run - m_new);
                m_run = m_new;
                l_run *= scale;
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            if (ALIBI) {
#pragma unroll
                for (int b = 0; b < kTB; ++b) bk[b] = mu - bk[b];
            }
            // P = 2^(S - m) as bf16 pairs over the first 64 columns of S_t
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
            tc::st32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::st32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            l_run += ls0 + ls1;
            if (k > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t o[32];
                    tc::ld32(tO + 32 * c, o);
                    tc::wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * scale);
                    tc::st32(tO + 32 * c, o);
                }
            }
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (leader) mbar_arrive(&bars[B_PFULL + t]);
            ++k;
        }
        // ------------------------------------------------------------ this stream's split partial
        bool have = ok && k > 0;
        if (have) have = wwait(&bars[B_ODONE + t], (k - 1) & 1, abort_flag, p.d_status);
        if (have) tc::fence_after_sync();
        const size_t part = (static_cast<size_t>(r) * p.hkv + kvh) * p.n_splits + 2 * split + t;
        float4 *wo = reinterpret_cast<float4 *>(p.ws_acc + (part * G + lane) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            uint32_t ob[32];
            if (have) {
                tc::ld32(tO + 32 * c, ob);
                tc::wait_ld();
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) ob[e] = 0u;
            }
            if (lane < G) {
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    wo[8 * c + v] = make_float4(__uint_as_float(ob[4 * v]), __uint_as_float(ob[4 * v + 1]),
                                                __uint_as_float(ob[4 * v + 2]), __uint_as_float(ob[4 * v + 3]));
            }
        }
        if (lane < G) {
            p.ws_ml[(part * G + lane) * 2 + 0] = have ? m_run : -INFINITY;
            p.ws_ml[(part * G + lane) * 2 + 1] = have ? l_run : 0.f;
        }
    }

    // ================================================================ teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 3) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, 512);
    }
}

template <int MODE>
cudaError_t launch_tc(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8, const CUtensorMap &tv8,
                      const AttnParams &p, cudaStream_t s) {
    auto kern = decode_tc_kernel<MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTc);
    if (e != cudaSuccess) return e;
    // two partials (softmax streams) per CTA
    dim3 grid(p.n_splits / 2, p.hkv, p.num_req);
    kern<<<grid, kThreadsTc, kSmemTc, s>>>(tk, tv, tk8, tv8, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_decode_combine(p, s);
}

}  // namespace

cudaError_t launch_decode_tc(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                             const CUtensorMap &tv8, const AttnParams &p, bool plain, cudaStream_t s) {
    if (plain) return launch_tc<1>(tk, tv, tk8, tv8, p, s);
    return p.alibi ? launch_tc<2>(tk, tv, tk8, tv8, p, s) : launch_tc<0>(tk, tv, tk8, tv8, p, s);
}

}  // namespace lazy
