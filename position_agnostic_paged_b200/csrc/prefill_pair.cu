// prefill_pair.cu -- causal prefill attention over the paged pool with deferred
// RoPE, on pairs of SMs: 2-SM tcgen05 MMAs (cta_group::2) with the query tile
// and the score tiles in tensor memory, K/V halves staged by TMA.
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Prefilling -- cached keys are read as stored and rotated
// once, by the distance between the query position and the document's
// offset, instead of being taken back to position 0 and rotated again; the
// phase is bound by compute.
//
// Where the one relative rotation goes.  Keys sit in the pool rotated at their
// local index j, so a score of query i (position p_i) and key j of a segment
// at offset o needs the angle (p_i - o - j).  This kernel rotates the QUERY
// tile, once per segment, by (P0 - o) on top of a first rotation by
// (p_i - P0) made once per CTA (P0 = the unit's first query position):
//   Q'_seg,i = R(P0 - o) R(p_i - P0) q_i = R(p_i - o) q_i,
// and uses every K tile exactly as stored.  A segment is a run of K tiles with
// one offset (a document: 512 tokens = 4 tiles of 128 keys), so the extra
// work is one rotation of the query rows per document instead of one rotation
// of every K tile; it runs in its own warpgroup into a second query buffer
// while the tensor core works on the previous document.  The materialised
// comparison path (keys rotated at absolute positions) is the same kernel
// with the query rotated once by p_i and no per-segment step; the ALiBi mode
// rotates nothing and adds the bias in the softmax.
//
// Work unit = 256 query rows (token, head-in-group pairs) of one KV head of one
// request, run by a cluster of two CTAs on two SMs: CTA rank r holds rows
// 128r .. 128r+127.  Each 2-SM MMA computes 256 rows; its B operand is split
// between the pair (K tile: keys 0-63 in CTA 0, 64-127 in CTA 1; V tile:
// head-dim columns 0-63 in CTA 0, 64-127 in CTA 1), so each SM loads and
// stores half of every K/V tile and the pair reads each tile from L2 once.
//
// Tensor memory (512 columns, the same layout in both CTAs):
//   Q'0 [0,64)  Q'1 [64,128)   query rows for even / odd segments (bf16 pairs)
//   S0 [128,256) S1 [256,384)  scores of even / odd K tiles (P over the first 64)
//   O  [384,512)               output accumulator
// With S double-buffered the MMA issuer computes S(j+1) while the softmax
// works on S(j); the softmax runs back to back over the tiles.
//
// Warps (384 threads per CTA):
//   warp 0      table walk (tile information ring) and K-half loads
//   warp 1      MMA issuer (rank 0 only) and tensor-memory allocation (both)
//   warp 2      V-half loads
//   warp 3      idle
//   warps 4-7   softmax, one thread per row of this CTA
//   warps 8-11  query rotations: the per-CTA query rows R(p_i - P0) q_i into
//               shared memory at the start, then per segment R(P0 - o) of them
//               into the segment's tensor-memory query buffer
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lazy {

namespace {

constexpr int kUnitRows = 256;                 // query rows per work unit (cluster)
constexpr int kCtaRows = 128;                  // rows per CTA
constexpr int kTileBlocks = 8;                 // 16-token blocks per K/V tile (128 keys)
constexpr int kHalfStage = 16384;              // one CTA's half of a K or V tile
constexpr int kKStages = 6, kVStages = 5, kInfoStages = 12;
constexpr int kThreads = 384;

struct PairTileInfo {
    uint32_t blk[kTileBlocks];
    uint32_t meta[kTileBlocks];
    int n;       // blocks in the tile (1..8); 0 marks the end of the walk
    int off;     // the segment's logical offset
    int flags;   // kFull: every key of the tile is visible to every row of the unit
    int seg;     // segment index (query buffer seg & 1)
};
constexpr int kFull = 1;

// shared memory layout (offsets from a 1024-aligned base)
constexpr int kOffQ0 = 0;                                       // 128 rows x 256 B, chunk-swizzled
constexpr int kOffK = kOffQ0 + kCtaRows * 256;                  // K half-stages
constexpr int kOffV = kOffK + kKStages * kHalfStage;            // V half-stages
constexpr int kOffInfo = kOffV + kVStages * kHalfStage;
constexpr int kRing = 128;                                      // table words / metadata in the walk ring
constexpr int kOffRing = kOffInfo + kInfoStages * static_cast<int>(sizeof(PairTileInfo));
constexpr int kOffBar = kOffRing + 2 * kRing * 4;
constexpr int B_KFULL = 0, B_KEMPTY = B_KFULL + kKStages, B_VFULL = B_KEMPTY + kKStages,
              B_VEMPTY = B_VFULL + kVStages, B_IFULL = B_VEMPTY + kVStages, B_IEMPTY = B_IFULL + kInfoStages,
              B_SFULL = B_IEMPTY + kInfoStages, B_PREADY = B_SFULL + 2, B_ODONE = B_PREADY + 2,
              B_OFINAL = B_ODONE + 1, B_QREADY = B_OFINAL + 1, B_QFREE = B_QREADY + 2, B_DRAIN = B_QFREE + 2,
              kNumBars = B_DRAIN + 1;
constexpr int kOffTheta = kOffBar + kNumBars * 8;
constexpr int kOffCS = kOffTheta + kHalfDim * 8;                // 2 x (64 cos, 64 sin) floats
constexpr int kOffMisc = kOffCS + 2 * 2 * kHalfDim * 4;
constexpr int kOffSlope = kOffMisc + 16;
constexpr int kSmemUse = kOffSlope + 32 * 4;
constexpr size_t kPairSmem = kSmemUse + 1024;
static_assert(kPairSmem <= 232448, "shared memory budget");
static_assert(sizeof(PairTileInfo) == 80, "tile info layout");

// tensor-memory column offsets
constexpr uint32_t TM_Q = 0, TM_S = 128, TM_O = 384;

constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays below 2^8 between rescales
// kPolyOf8 pairs of scores in every 8 take their exponentials on the FMA pipe (exp2_poly2),
// the rest on the SFU: with every exponential on the SFU the softmax of a tile takes longer
// than the tensor core's MMAs on it (measured on B200: about 11.5 cycles per warp-wide ex2).
constexpr int kPolyOf8 = 4;

// Register split (launch: 384 threads x 168 registers): the loader/MMA warpgroup gives up
// registers to the softmax (the whole 128-score row lives in registers) and the rotations.
constexpr int kLaunchRegs = 168, kLoadRegs = 72, kSoftmaxRegs = 248, kRotRegs = 184;
static_assert(128 * (kLoadRegs + kSoftmaxRegs + kRotRegs) <= kThreads * kLaunchRegs, "register split");
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(N)); }

// MODE: kLazy (pool keys as stored, query rotated per segment), kPlain (keys from a
// materialised copy indexed by table position, query rotated once at absolute positions),
// kAlibi (pool keys as stored, nothing rotated, ALiBi bias in the softmax).
constexpr int kLazy = 0, kPlain = 1, kAlibi = 2;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ uint32_t cta_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Shared::cluster address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_rank(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}
// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA).  The
// data these arrivals publish lives in tensor memory and is ordered by tcgen05 fences around
// the synchronisation, so the arrive keeps the default CTA-scope release: a cluster-scope
// release measured about 870 cycles on B200 (against 8 for a local arrive), on the softmax's
// critical path once per tile.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool try_wait_cluster(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait on a barrier that threads of the peer CTA arrive on.
__device__ __forceinline__ bool wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *d_status) {
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (try_wait_cluster(bar, parity)) return true;
        if ((i & 255) == 255 && *abort_flag) return false;
    }
    *abort_flag = 1;
    set_status(d_status, LAZY_DSTATUS_TIMEOUT);
    return false;
}
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *d_status) {
    const bool ok = wait_or_abort(bar, parity, abort_flag, d_status);
    return __all_sync(0xffffffffu, ok);
}
// Same decision for the 128 threads of one warpgroup (named barrier `id`).
__device__ __forceinline__ bool group_all(bool ok, int id) {
    uint32_t any_fail;
    asm volatile(
        "{\n .reg .pred p, q;\n setp.eq.u32 p, %1, 0;\n barrier.cta.red.or.pred q, %2, 128, p;\n"
        " selp.u32 %0, 1, 0, q;\n}\n"
        : "=r"(any_fail)
        : "r"(ok ? 1u : 0u), "r"(id)
        : "memory");
    return any_fail == 0;
}
__device__ __forceinline__ void group_sync(int id) { asm volatile("barrier.cta.sync %0, 128;" ::"r"(id) : "memory"); }

// 2D / 4D tiled loads of this CTA's half into its own shared memory, completing on the
// mbarrier at shared::cluster address `mbar` (the cluster's rank-0 barrier): the 2-SM form,
// without multicast.
__device__ __forceinline__ void tma2_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tma2_load_4d(void *dst, const CUtensorMap *map, int x, int y, int h, int b,
                                             uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(h), "r"(b), "r"(mbar)
        : "memory");
}

// ------------------------------------------------------------------ 2-SM tensor-core helpers
__device__ __forceinline__ void tmem_alloc2(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols));
}
__device__ __forceinline__ void tmem_relinquish2() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc2(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}
// D[tmem] (+)= A[tmem] * B[smem], 256 rows over the pair
__device__ __forceinline__ void mma2_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}
// Arrives once on the mbarrier at the same offset in both CTAs of the pair when every MMA
// issued before it has completed.
__device__ __forceinline__ void commit2_both(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(static_cast<uint16_t>(3))
        : "memory");
}
__device__ __forceinline__ void commit2_self(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// MMA issuer: S(t) = Q'_seg(t) K(t)^T into S buffer t & 1 (2-SM MMAs, 256 rows by 128 keys).
// Returns the tile's block count once its MMAs are issued, 0 at the end of the tiles (the
// end-of-walk entry), -1 when a wait ran out.  The tile's information entry stays held (the
// caller releases it after PV(t)).  At the first tile of a segment the previous segment's query
// buffer is released (its last S MMAs are the commit's predecessors) and the new segment's
// query rows are awaited.
__device__ __forceinline__ int issue_s_tile(int t, int &cur_seg, uint64_t *bars, const PairTileInfo *info,
                                            volatile int *abort_flag, int *d_status, uint32_t tbase, uint64_t dK0,
                                            uint32_t idq) {
    const int is = t % kInfoStages;
    if (!wait_or_abort(&bars[B_IFULL + is], (t / kInfoStages) & 1, abort_flag, d_status)) return -1;
    const int n = info[is].n, seg = info[is].seg;
    if (n == 0) return 0;
    if (seg != cur_seg) {
        if (cur_seg >= 0) commit2_both(&bars[B_QFREE + (cur_seg & 1)]);
        cur_seg = seg;
        if (!wait_cluster(&bars[B_QREADY + (seg & 1)], (seg >> 1) & 1, abort_flag, d_status)) return -1;
    }
    const int ks = t % kKStages;
    if (!wait_or_abort(&bars[B_KFULL + ks], (t / kKStages) & 1, abort_flag, d_status)) return -1;
    tc::fence_after_sync();
    const uint32_t tS = tbase + TM_S + 128 * (t & 1);
    const uint32_t tQ = tbase + TM_Q + 64 * (seg & 1);
    const uint64_t kb = dK0 + static_cast<uint64_t>((ks * kHalfStage) >> 4);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
        const uint64_t o = static_cast<uint64_t>(((kk >> 2) * (kHalfStage / 2) + (kk & 3) * 32) >> 4);
        mma2_ts(tS, tQ + 8 * kk, kb + o, idq, kk > 0 ? 1u : 0u);
    }
    commit2_both(&bars[B_SFULL + (t & 1)]);
    commit2_both(&bars[B_KEMPTY + ks]);
    return n;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) prefill_pair_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                   const __grid_constant__ CUtensorMap tmV,
                                                                   const __grid_constant__ CUtensorMap tmK4,
                                                                   const __grid_constant__ CUtensorMap tmV8,
                                                                   const AttnParams p) {
    constexpr bool PLAIN = MODE == kPlain;
    constexpr bool LAZY = MODE == kLazy;
    constexpr bool ALIBI = MODE == kAlibi;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    PairTileInfo *info = reinterpret_cast<PairTileInfo *>(sm + kOffInfo);
    double *theta_s = reinterpret_cast<double *>(sm + kOffTheta);
    float *cs_s = reinterpret_cast<float *>(sm + kOffCS);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    float *slope_s = reinterpret_cast<float *>(sm + kOffSlope);

    const uint32_t rank = cta_rank();
    // work unit (m-tile, KV head, request) of this cluster and the part of its keys it takes
    int unit = static_cast<int>(blockIdx.x >> 1), part = -1;
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
    const int R0 = mt * kUnitRows;
    // uniform over the cluster: a unit without rows does nothing (both CTAs leave together)
    if (R0 >= T * G) return;
    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    const int wbeg = part == 1 ? n_words / 2 : 0, wend = part == 0 ? n_words / 2 : n_words;
    const uint32_t *tbl = p.table + wbase;
    const int pos0 = p.q_pos0[r];
    const int tok_first = R0 / G;
    const int tok_last = min(T - 1, (R0 + kUnitRows - 1) / G);
    const int Pbase = pos0 + tok_first;   // smallest query position of the unit
    const int Pmax = pos0 + tok_last;     // largest query position of the unit

    // consumers of one tile-information entry: the V producer, the softmax warps, the MMA
    // issuer (rank 0) and, on the lazy path, the rotation warps
    const uint32_t info_consumers = 1 + 4 + (rank == 0 ? 1 : 0) + (LAZY ? 4 : 0);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kKStages; ++i) {
            mbar_init(&bars[B_KFULL + i], 1);
            mbar_init(&bars[B_KEMPTY + i], 1);
        }
        for (int i = 0; i < kVStages; ++i) {
            mbar_init(&bars[B_VFULL + i], 1);
            mbar_init(&bars[B_VEMPTY + i], 1);
        }
        for (int i = 0; i < kInfoStages; ++i) {
            mbar_init(&bars[B_IFULL + i], 1);
            mbar_init(&bars[B_IEMPTY + i], info_consumers);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bars[B_SFULL + b], 1);
            mbar_init(&bars[B_PREADY + b], 8);   // 4 softmax warps x 2 CTAs
            mbar_init(&bars[B_QREADY + b], 8);   // 4 rotation warps x 2 CTAs
            mbar_init(&bars[B_QFREE + b], 1);
        }
        mbar_init(&bars[B_ODONE], 1);
        mbar_init(&bars[B_OFINAL], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        if (rank == 0 && mt == 0 && kvh == 0 && part <= 0 && n_words > p.max_words)
            set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (threadIdx.x < kHalfDim) theta_s[threadIdx.x] = p.rope.theta[threadIdx.x];
    if (ALIBI && threadIdx.x < G) slope_s[threadIdx.x] = p.alibi_log2[kvh * G + threadIdx.x];
    if (warp == 1) {
        tmem_alloc2(tmem_slot, 512);
        tmem_relinquish2();
    }
    tc::fence_before_sync();
    __syncthreads();
    cluster_sync_all();   // barrier inits and the allocation are visible across the pair
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;

    if (warp < 4) {
    setmaxnreg_dec<kLoadRegs>();
    if (warp == 0) {
        // ============================================================ table walk + K halves
        // The table words and their blocks' metadata are fetched 32 at a time, one per lane of
        // the warp, into a ring in shared memory two batches ahead of the tiles lane 0 forms and
        // loads: every global load of the walk is in flight while earlier tiles are issued,
        // instead of two dependent round trips per tile.
        uint32_t *ring_w = reinterpret_cast<uint32_t *>(sm + kOffRing);
        uint32_t *ring_m = ring_w + kRing;
        const int nw = wend - wbeg;
        auto ld_word = [&](int i) -> uint32_t { return i < nw ? tbl[wbeg + i] : 0xFFFFFFFFu; };
        auto ld_meta = [&](uint32_t w, int i) -> uint32_t {
            const uint32_t b = word_block(w);
            return (i < nw && b < static_cast<uint32_t>(p.num_blocks)) ? p.blk_meta[b] : 0u;
        };
        {
            const uint32_t w0 = ld_word(lane);
            ring_m[lane] = ld_meta(w0, lane);
            ring_w[lane] = w0;
            ring_w[32 + lane] = ld_word(32 + lane);
        }
        __syncwarp();
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmK4);
        }
        int j = 0, seg = -1, prev_off = INT_MIN, cur = 0;
        bool stop = false;
        for (int k = 0; 32 * k < nw && !stop; ++k) {
            // in flight during this batch: the metadata of batch k + 1, the words of batch k + 2
            const int i1 = 32 * (k + 1) + lane, i2 = 32 * (k + 2) + lane;
            const uint32_t m1 = ld_meta(ring_w[i1 % kRing], i1);
            const uint32_t w2 = ld_word(i2);
            if (lane == 0) {
                const int avail = min(32 * (k + 1), nw);   // words whose metadata is in the ring
                while (cur < nw && (cur + kTileBlocks <= avail || avail == nw)) {
                    // the tile: up to 8 consecutive words that share one offset
                    uint32_t wd[kTileBlocks], mt_k[kTileBlocks];
#pragma unroll
                    for (int q = 0; q < kTileBlocks; ++q) {
                        const bool in = cur + q < nw;
                        wd[q] = in ? ring_w[(cur + q) % kRing] : 0xFFFFFFFFu;
                        mt_k[q] = in ? ring_m[(cur + q) % kRing] : 0u;
                    }
                    const int off = word_offset(wd[0]);
                    int n = 1;
#pragma unroll
                    for (int q = 1; q < kTileBlocks; ++q)
                        if (n == q && cur + q < nw && word_offset(wd[q]) == off) n = q + 1;
                    const int w0 = wbeg + cur;   // word index inside the request's table
                    cur += n;
                    bool full = n == kTileBlocks;
                    int kmin = INT_MAX;   // smallest key position of the tile
#pragma unroll
                    for (int q = 0; q < kTileBlocks; ++q) {
                        const bool ok = q < n && word_block(wd[q]) < static_cast<uint32_t>(p.num_blocks);
                        if (!ok) mt_k[q] = 0u;
                        if (q < n && !ok) set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
                        if (ok && meta_valid(mt_k[q]) > 0) kmin = min(kmin, off + meta_j0(mt_k[q]));
                        full = full && meta_valid(mt_k[q]) == kBlockTokens &&
                               off + meta_j0(mt_k[q]) + kBlockTokens - 1 <= Pbase;
                    }
                    // a tile no query of the unit can see is left out (the same decision in both CTAs)
                    if (kmin > Pmax) continue;
                    if (LAZY && off != prev_off) {
                        ++seg;
                        prev_off = off;
                    }
                    const int is = j % kInfoStages;
                    if (!wait_or_abort(&bars[B_IEMPTY + is], ((j / kInfoStages) & 1) ^ 1, abort_flag, p.d_status)) {
                        stop = true;
                        break;
                    }
                    PairTileInfo &ti = info[is];
#pragma unroll
                    for (int q = 0; q < kTileBlocks; ++q) {
                        ti.blk[q] = q < n ? word_block(wd[q]) : 0u;
                        ti.meta[q] = mt_k[q];
                    }
                    ti.n = n;
                    ti.off = off;
                    ti.flags = full ? kFull : 0;
                    ti.seg = LAZY ? seg : 0;
                    mbar_arrive(&bars[B_IFULL + is]);
                    // this CTA's half of the K tile: blocks 4*rank .. 4*rank+3 (keys 64*rank ..)
                    const int ks = j % kKStages;
                    if (!wait_or_abort(&bars[B_KEMPTY + ks], ((j / kKStages) & 1) ^ 1, abort_flag, p.d_status)) {
                        stop = true;
                        break;
                    }
                    const uint32_t full_bar = map_rank(&bars[B_KFULL + ks], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&bars[B_KFULL + ks], static_cast<uint32_t>(n) * kBlockBytes);
                    uint8_t *kd = sm + kOffK + ks * kHalfStage;
                    const int k0 = 4 * static_cast<int>(rank);
                    const int nh = max(0, min(4, n - k0));   // blocks of this half that exist
                    bool contig = nh == 4;
#pragma unroll
                    for (int q = 1; q < 4; ++q)
                        contig = contig && word_block(wd[k0 + q]) == word_block(wd[k0]) + static_cast<uint32_t>(q);
                    contig = contig && (PLAIN || word_block(wd[k0]) + 4u <= static_cast<uint32_t>(p.num_blocks));
                    if (contig) {
                        const int z = PLAIN ? wbase + w0 + k0 : static_cast<int>(word_block(wd[k0]));
                        tma2_load_4d(kd, &tmK4, 0, 0, kvh, z, full_bar);
                        tma2_load_4d(kd + kHalfStage / 2, &tmK4, kHalfDim, 0, kvh, z, full_bar);
                    } else {
                        for (int q = 0; q < nh; ++q) {
                            const uint32_t b = word_block(wd[k0 + q]);
                            int row;
                            if (b >= static_cast<uint32_t>(p.num_blocks))
                                row = p.k_rows;   // fully out of bounds: the box is zero-filled
                            else
                                row = PLAIN ? ((wbase + w0 + k0 + q) * p.hkv + kvh) * kBlockTokens
                                            : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                            tma2_load_2d(kd + q * kBoxBytes, &tmK, 0, row, full_bar);
                            tma2_load_2d(kd + kHalfStage / 2 + q * kBoxBytes, &tmK, kHalfDim, row, full_bar);
                        }
                    }
                    ++j;
                }
            }
            cur = __shfl_sync(0xffffffffu, cur, 0);
            j = __shfl_sync(0xffffffffu, j, 0);
            stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
            ring_m[i1 % kRing] = m1;
            ring_w[i2 % kRing] = w2;
            __syncwarp();
        }
        // end of the walk
        if (lane == 0 && !stop) {
            const int is = j % kInfoStages;
            if (wait_or_abort(&bars[B_IEMPTY + is], ((j / kInfoStages) & 1) ^ 1, abort_flag, p.d_status)) {
                info[is].n = 0;
                mbar_arrive(&bars[B_IFULL + is]);
            }
        }
    } else if (warp == 2) {
        // ============================================================ V halves (head-dim columns 64*rank ..)
        if (lane == 0) {
            tma_prefetch_desc(&tmV);
            tma_prefetch_desc(&tmV8);
            for (int j = 0;; ++j) {
                const int is = j % kInfoStages;
                if (!wait_or_abort(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status)) break;
                const int n = info[is].n;
                uint32_t blk[kTileBlocks];
#pragma unroll
                for (int k = 0; k < kTileBlocks; ++k) blk[k] = info[is].blk[k];
                mbar_arrive(&bars[B_IEMPTY + is]);
                if (n == 0) break;
                const int vs = j % kVStages;
                if (!wait_or_abort(&bars[B_VEMPTY + vs], ((j / kVStages) & 1) ^ 1, abort_flag, p.d_status)) break;
                const uint32_t full_bar = map_rank(&bars[B_VFULL + vs], 0);
                if (rank == 0) mbar_arrive_expect_tx(&bars[B_VFULL + vs], static_cast<uint32_t>(n) * kBlockBytes);
                uint8_t *vd = sm + kOffV + vs * kHalfStage;
                const int x = kHalfDim * static_cast<int>(rank);
                bool contig = n == kTileBlocks && blk[0] + static_cast<uint32_t>(kTileBlocks) <=
                                                      static_cast<uint32_t>(p.num_blocks);
#pragma unroll
                for (int k = 1; k < kTileBlocks; ++k) contig = contig && blk[k] == blk[0] + static_cast<uint32_t>(k);
                if (contig) {
                    tma2_load_4d(vd, &tmV8, x, 0, kvh, static_cast<int>(blk[0]), full_bar);
                } else {
                    for (int k = 0; k < n; ++k) {
                        const int row = blk[k] >= static_cast<uint32_t>(p.num_blocks)
                                            ? p.v_rows
                                            : (static_cast<int>(blk[k]) * p.hkv + kvh) * kBlockTokens;
                        tma2_load_2d(vd + k * kBoxBytes, &tmV, x, row, full_bar);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer (rank 0)
        if (rank == 0 && lane == 0) {
            const uint32_t idq = tc::idesc_bf16(256, 128, false);
            const uint32_t idv = tc::idesc_bf16(256, 128, true);
            const uint64_t dK0 = tc::smem_desc(smem_u32(sm + kOffK), 16, 1024);
            const uint64_t dV0 = tc::smem_desc(smem_u32(sm + kOffV), 16, 1024);
            const uint32_t tO = tbase + TM_O;
            int cur_seg = -1;
            // blocks of tile t (S issued, PV next) and of tile t + 1 (S issued); 0 = no such tile
            int na = issue_s_tile(0, cur_seg, bars, info, abort_flag, p.d_status, tbase, dK0, idq);
            int nb = na > 0 ? issue_s_tile(1, cur_seg, bars, info, abort_flag, p.d_status, tbase, dK0, idq) : na;
            bool ok = na >= 0 && nb >= 0;
            int t = 0;
            for (; ok && na > 0; ++t) {
                // O += P(t) V(t): P(t) over the first 64 columns of S buffer t & 1
                if (!wait_cluster(&bars[B_PREADY + (t & 1)], (t >> 1) & 1, abort_flag, p.d_status)) {
                    ok = false;
                    break;
                }
                const int vs = t % kVStages;
                if (!wait_or_abort(&bars[B_VFULL + vs], (t / kVStages) & 1, abort_flag, p.d_status)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                const uint32_t tP = tbase + TM_S + 128 * (t & 1);
                const uint64_t vb = dV0 + static_cast<uint64_t>((vs * kHalfStage) >> 4);
                for (int k = 0; k < na; ++k)
                    mma2_ts(tO, tP + 8 * k, vb + static_cast<uint64_t>((k * kBoxBytes) >> 4), idv,
                            (t > 0 || k > 0) ? 1u : 0u);
                commit2_both(&bars[B_ODONE]);
                commit2_both(&bars[B_VEMPTY + vs]);
                mbar_arrive(&bars[B_IEMPTY + t % kInfoStages]);   // info entry t released
                // S(t+2) reuses S buffer t & 1: issued after PV(t), which read P(t) there
                const int nc = nb > 0 ? issue_s_tile(t + 2, cur_seg, bars, info, abort_flag, p.d_status, tbase, dK0, idq)
                                      : 0;
                if (nc < 0) {
                    ok = false;
                    break;
                }
                na = nb;
                nb = nc;
            }
            // the end-of-walk entry is released too: it is entry t once no tile is left
            if (ok) mbar_arrive(&bars[B_IEMPTY + t % kInfoStages]);
            // the softmax warps' epilogue reads O once every PV has completed
            commit2_both(&bars[B_OFINAL]);
            // every MMA issued has completed before tensor memory is released
            commit2_self(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    }
    } else if (warp < 8) {
        // ============================================================ softmax (one row per thread)
        setmaxnreg_inc<kSoftmaxRegs>();
        const int row = threadIdx.x - 128;                 // 0..127 in this CTA
        const int R = R0 + kCtaRows * static_cast<int>(rank) + row;
        const bool row_ok = R < T * G;
        const int tok = row_ok ? R / G : tok_first;
        const int g = R % G;
        const int prow = pos0 + tok;
        const float slope = ALIBI ? slope_s[g] : 0.f;
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        const uint32_t pready0 = map_rank(&bars[B_PREADY], 0), pready1 = map_rank(&bars[B_PREADY + 1], 0);
        const uint32_t tO = tbase + TM_O;
        float m_run = -INFINITY, l_run = 0.f;
        int j = 0;
        bool ok = true;
        for (;; ++j) {
            const int is = j % kInfoStages;
            if (!warp_wait(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status)) {
                ok = false;
                break;
            }
            const PairTileInfo &ti = info[is];
            const int n = ti.n;
            const bool full = (ti.flags & kFull) != 0;
            int lim[kTileBlocks];
            float bk[kTileBlocks];
#pragma unroll
            for (int k = 0; k < kTileBlocks; ++k) {
                const int nv = k < n ? meta_valid(ti.meta[k]) : 0;
                lim[k] = max(0, min(nv, prow - ti.off - meta_j0(ti.meta[k]) + 1));
                bk[k] = ALIBI ? slope * static_cast<float>(ti.off + meta_j0(ti.meta[k]) - prow) : 0.f;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_IEMPTY + is]);
            if (n == 0) break;
            if (!warp_wait(&bars[B_SFULL + (j & 1)], (j >> 1) & 1, abort_flag, p.d_status)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const uint32_t tS = tbase + TM_S + 128 * (j & 1);
            uint32_t sv[128];
            tc::ld32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::ld32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            tc::ld32(tS + lane_off + 64, *reinterpret_cast<uint32_t(*)[32]>(sv + 64));
            tc::ld32(tS + lane_off + 96, *reinterpret_cast<uint32_t(*)[32]>(sv + 96));
            tc::wait_ld();
            if (ALIBI) {
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
                for (int c = 0; c < 128; ++c) sv[c] = (c & 15) < lim[c >> 4] ? sv[c] : 0xFF800000u;
            }
            auto f = [&](int c) { return __uint_as_float(sv[c]); };
            float m0 = f(0), m1 = f(1);
            if (ALIBI) {
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
            if (ALIBI) {
#pragma unroll
                for (int k = 0; k < kTileBlocks; ++k) bk[k] = mu - bk[k];
            }
            float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
            for (int e = 0; e < 64; ++e) {
                const float nmo = -(ALIBI ? bk[e >> 3] : mu);
                float x0 = f(2 * e), x1 = f(2 * e + 1);
                add2(x0, x1, nmo, nmo);
                float p0, p1;
                if (e % 8 >= 8 - kPolyOf8) {
                    exp2_poly2(x0, x1, p0, p1);
                } else {
                    p0 = fast_exp2(x0);
                    p1 = fast_exp2(x1);
                }
                add2(ls0, ls1, p0, p1);
                sv[e] = pack_bf16(p0, p1);
            }
            tc::st32(tS + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(sv + 0));
            tc::st32(tS + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
            l_run += ls0 + ls1;
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // O holds P(j-1) V(j-1) only once PV(j-1) has completed (it was issued after S(j))
                if (!warp_wait(&bars[B_ODONE], (j - 1) & 1, abort_flag, p.d_status)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
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
            if (lane == 0) mbar_arrive_cluster((j & 1) ? pready1 : pready0);
        }
        // ------------------------------------------------------------ epilogue
        bool have = ok && j > 0;
        if (have) have = warp_wait(&bars[B_OFINAL], 0, abort_flag, p.d_status);
        // a row that saw no key keeps m_run = -inf (its polynomial exponentials of masked scores
        // are tiny but not zero, so l alone does not tell)
        const float inv = (have && m_run != -INFINITY && l_run > 0.f) ? 1.f / l_run : 0.f;
        const bool all_have = __all_sync(0xffffffffu, have);
        if (all_have) tc::fence_after_sync();
        const int urow = kCtaRows * static_cast<int>(rank) + row;   // row inside the unit
        if (part >= 0) {
            // half of a split unit: unnormalised O, running max and sum (log2 domain) for the
            // combine step
            const size_t srow = static_cast<size_t>((unit - p.pf_base) * 2 + part) * kUnitRows + urow;
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
            const bool seen = have && m_run != -INFINITY;
            p.ws_ml[2 * srow] = seen ? m_run : -INFINITY;
            p.ws_ml[2 * srow + 1] = seen ? l_run : 0.f;
        }
        uint4 *o = (row_ok && part < 0)
                       ? reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(q0 + tok) * p.hq + kvh * G + g) * kHeadDim)
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
        // ============================================================ query rotations
        setmaxnreg_inc<kRotRegs>();
        const int tid = threadIdx.x - 256;   // 0..127
        uint8_t *q0s = sm + kOffQ0;
        const uint32_t qready0 = map_rank(&bars[B_QREADY], 0), qready1 = map_rank(&bars[B_QREADY + 1], 0);
        // (1) this CTA's query rows rotated by (p_i - Pref) into shared memory (Pref = P0 on the
        // lazy path, 0 on the plain path; nothing is rotated under ALiBi, whose table is zero).
        // Thread (ch, rb) writes pairs 8ch..8ch+7 of rows rb + 16k; between rows rb + 16k and
        // rb + 16(k+1) the token advances by dlo = 16 / G or dlo + 1, so the angles advance by
        // rotations from two step tables.  Row i occupies 256 B, its 16-byte chunk c at
        // (c ^ (i & 7)) so that a warp reading one chunk of 32 consecutive rows is conflict-free.
        {
            const int ch = tid & 7, rb = tid >> 3;
            const int dlo = 16 / G;
            float cA[8], sA[8], cB[8], sB[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                rope_cos_sin(dlo, theta_s[8 * ch + e], cA[e], sA[e]);
                rope_cos_sin(dlo + 1, theta_s[8 * ch + e], cB[e], sB[e]);
            }
            const int qref = PLAIN ? 0 : Pbase;
            const int rowbase = R0 + kCtaRows * static_cast<int>(rank) + rb;   // unit row of k = 0
            int tk_prev = rowbase / G;
            float cc[8], ss[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) rope_cos_sin(pos0 + tk_prev - qref, theta_s[8 * ch + e], cc[e], ss[e]);
#pragma unroll 1
            for (int kg = 0; kg < 8; kg += 4) {
                uint4 a4[4], b4[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int Rr = rowbase + 16 * (kg + u);
                    a4[u] = make_uint4(0, 0, 0, 0);
                    b4[u] = make_uint4(0, 0, 0, 0);
                    if (Rr < T * G) {
                        const uint16_t *q = p.q_raw + (static_cast<size_t>(q0 + Rr / G) * p.hq + kvh * G + Rr % G) * kHeadDim;
                        a4[u] = *reinterpret_cast<const uint4 *>(q + 8 * ch);
                        b4[u] = *reinterpret_cast<const uint4 *>(q + kHalfDim + 8 * ch);
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int k = kg + u;
                    const int Rr = rowbase + 16 * k;
                    const int tk = Rr / G;
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
                    const int rw = rb + 16 * k;   // row in this CTA
                    *reinterpret_cast<uint4 *>(q0s + rw * 256 + ((ch ^ (rw & 7)) << 4)) = lo;
                    *reinterpret_cast<uint4 *>(q0s + rw * 256 + (((8 + ch) ^ (rw & 7)) << 4)) = hi;
                }
            }
        }
        group_sync(2);
        // (2) query rows into a tensor-memory query buffer: thread = row, rotated by (Pbase - o)
        // per segment on the lazy path, copied once otherwise
        const int row = tid;
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
        auto write_q = [&](int buf, const float *cs) {
            uint32_t qw[64];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 a4 = *reinterpret_cast<const uint4 *>(q0s + row * 256 + ((c ^ (row & 7)) << 4));
                const uint4 b4 = *reinterpret_cast<const uint4 *>(q0s + row * 256 + (((8 + c) ^ (row & 7)) << 4));
                const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4);
                const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if (cs) {
                        const int i0 = 8 * c + 2 * e;
                        const float a0 = bf16_lo(aw[e]), a1 = bf16_hi(aw[e]);
                        const float b0 = bf16_lo(bw[e]), b1 = bf16_hi(bw[e]);
                        const float c0 = cs[i0], c1 = cs[i0 + 1], s0 = cs[kHalfDim + i0], s1 = cs[kHalfDim + i0 + 1];
                        float ac0, ac1, bc0, bc1, lo0, lo1, hi0, hi1;
                        mul2(ac0, ac1, a0, a1, c0, c1);
                        mul2(bc0, bc1, b0, b1, c0, c1);
                        fma2v(lo0, lo1, -b0, -b1, s0, s1, ac0, ac1);
                        fma2v(hi0, hi1, a0, a1, s0, s1, bc0, bc1);
                        qw[4 * c + e] = pack_bf16(lo0, lo1);
                        qw[32 + 4 * c + e] = pack_bf16(hi0, hi1);
                    } else {
                        qw[4 * c + e] = aw[e];
                        qw[32 + 4 * c + e] = bw[e];
                    }
                }
            }
            const uint32_t tQ = tbase + TM_Q + 64 * buf;
            tc::st32(tQ + lane_off + 0, *reinterpret_cast<uint32_t(*)[32]>(qw + 0));
            tc::st32(tQ + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(qw + 32));
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(buf ? qready1 : qready0);
        };
        if (!LAZY) {
            write_q(0, nullptr);
        } else {
            int cur = -1;
            for (int j = 0;; ++j) {
                const int is = j % kInfoStages;
                const bool okw = wait_or_abort(&bars[B_IFULL + is], (j / kInfoStages) & 1, abort_flag, p.d_status);
                if (!group_all(okw, 3)) break;
                const int n = info[is].n, off = info[is].off, seg = info[is].seg;
                __syncwarp();
                if (lane == 0) mbar_arrive(&bars[B_IEMPTY + is]);
                if (n == 0) break;
                if (seg == cur) continue;
                cur = seg;
                const int buf = seg & 1;
                if (seg >= 2) {
                    // the buffer's previous segment (seg - 2) has had its last S MMA complete
                    const bool okf = wait_or_abort(&bars[B_QFREE + buf], ((seg - 2) >> 1) & 1, abort_flag, p.d_status);
                    if (!group_all(okf, 3)) break;
                    tc::fence_after_sync();
                }
                float *cs = cs_s + buf * 2 * kHalfDim;
                if (tid < kHalfDim) rope_cos_sin(Pbase - off, theta_s[tid], cs[tid], cs[kHalfDim + tid]);
                group_sync(2);
                write_q(buf, cs);
            }
        }
    }

    // ================================================================ teardown
    tc::fence_before_sync();
    __syncthreads();
    cluster_sync_all();   // no CTA leaves while the pair's MMAs may still use its memory
    if (warp == 1) {
        tc::fence_after_sync();
        tmem_dealloc2(tbase, 512);
    }
}

// Merges the two halves of each split unit: with M = max(m0, m1) and w_i = 2^(m_i - M),
// O = (w0 O0 + w1 O1) / (w0 l0 + w1 l1).  One warp per query row, 4 columns of d per lane.
__global__ void __launch_bounds__(256) prefill_pair_combine_kernel(const AttnParams p) {
    const int s = blockIdx.x, row_in = blockIdx.y * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    const int unit = p.pf_base + s;
    const int mt = unit % p.pf_mtiles, kvh = (unit / p.pf_mtiles) % p.hkv, r = unit / (p.pf_mtiles * p.hkv);
    const int G = p.group;
    const int q0 = p.cu_q[r], T = p.cu_q[r + 1] - q0;
    const int R = mt * kUnitRows + row_in;
    if (R >= T * G) return;
    const size_t r0 = static_cast<size_t>(2 * s) * kUnitRows + row_in, r1 = r0 + kUnitRows;
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

template <int MODE>
cudaError_t launch_pair_t(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk4,
                          const CUtensorMap &tv8, const AttnParams &p, cudaStream_t s) {
    auto kern = prefill_pair_kernel<MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem);
    if (e != cudaSuccess) return e;
    static_assert(kUnitRows == kPrefillRows, "rows per unit");
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (p.pf_base + 2 * p.pf_nsplit));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kPairSmem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, tk, tv, tk4, tv8, p);
    if (e != cudaSuccess || p.pf_nsplit == 0) return e;
    prefill_pair_combine_kernel<<<dim3(p.pf_nsplit, kUnitRows / 8), 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_pair(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk4,
                                const CUtensorMap &tv8, const AttnParams &p, bool plain, cudaStream_t s) {
    if (plain) return launch_pair_t<kPlain>(tk, tv, tk4, tv8, p, s);
    return p.alibi ? launch_pair_t<kAlibi>(tk, tv, tk4, tv8, p, s) : launch_pair_t<kLazy>(tk, tv, tk4, tv8, p, s);
}

}  // namespace lazy
