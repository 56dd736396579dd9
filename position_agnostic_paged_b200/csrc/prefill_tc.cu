// prefill_tc.cu -- causal prefill attention over the paged pool with deferred
// RoPE on the fifth-generation tensor cores (tcgen05.mma, accumulators in
// tensor memory, operands staged by TMA).
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Prefilling -- the kernel loads cached KV blocks and applies
// one relative rotation based on the offset between the query and the cached
// document instead of resetting the keys to position 0 and rotating them
// again; the attention is compute-bound.
//
// Where the single relative rotation goes.  Keys sit in the pool rotated at
// their local index j.  For a query tile whose first token is at position P,
// the rotation warpgroup keeps Qt = R(p_i - P) q_i (once per CTA, bf16 in
// shared memory).  Each time the table walk enters a segment with offset o it
// writes Q' = R(P - o) Qt into one of two query buffers: one relative
// rotation by (P - o), uniform across the tile, so scores carry the angle
// (p_i - o - j) of eager RoPE attention.  Stored keys go from TMA to the
// tensor core untouched, and the rotation overlaps the MMAs of the previous
// segment.
//
// CTA = one 128-row query tile (rows are (token, head-in-group) pairs,
// token-major) of one KV head of one request; 12 warps:
//   warp 0       TMA producer: per KV tile (<= 8 blocks = 128 keys of one
//                segment) the K and V boxes into double-buffered stages
//   warp 1       tensor-memory owner and MMA issuer: S = Q' K^T (8 MMAs,
//                K = 16 each) into S[j%2], then O += P V (one MMA per block)
//   warps 2-3    idle
//   warps 4-7    softmax, one thread per query row: S row from tensor memory,
//                mask, online softmax with lazy rescaling of O, P (bf16) back
//                to tensor memory; the epilogue writes O / l
//   warps 8-11   query rotation (Qt once, then Q' per segment)
// Tensor memory (512 columns): S0 [0,128) S1 [128,256) O [256,384)
// P0 [384,448) P1 [448,512).
#include <climits>

#include "common.cuh"
#include "kernels.h"
#include "tc.cuh"

namespace lazy {

namespace {

constexpr int kRows = 128;
constexpr int kTileBlocks = 8;
constexpr int kTileBytes = kRows * kHeadDim * 2;   // 32 KiB
constexpr int kHalfPlane = kTileBytes / 2;         // 16 KiB
constexpr int kThreads = 384;

constexpr int kOffQt = 0;
constexpr int kOffQ = kOffQt + kTileBytes;
constexpr int kOffK = kOffQ + 2 * kTileBytes;
constexpr int kOffV = kOffK + 2 * kTileBytes;
constexpr int kOffBar = kOffV + 2 * kTileBytes;
constexpr int kNumBars = 21;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kOffSeg = kOffMisc + 16;
constexpr int kOffTheta = kOffSeg + kHalfDim * 8;
constexpr int kSmemUse = kOffTheta + kHalfDim * 8;
constexpr size_t kTcSmem = kSmemUse + 1024;
static_assert(kTcSmem <= 232448, "shared memory budget");

// barrier indices
constexpr int B_KFULL = 0, B_KEMPTY = 2, B_VFULL = 4, B_VEMPTY = 6, B_SFULL = 8, B_SFREE = 10, B_PFULL = 12,
              B_ODONE = 14, B_QFULL = 16, B_QEMPTY = 18, B_DRAIN = 20;

constexpr float kRescaleThreshold = 8.0f;   // log2 units: P stays below 2^8 between rescales

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

struct KTile {
    int n;     // blocks in the tile (1..8), all from one segment
    int off;   // the segment's logical offset
};

// Tiles are formed identically by every role: up to 8 consecutive table words
// that share one offset (a tile never spans two segments).
__device__ __forceinline__ KTile ktile(const uint32_t *tbl, int w, int n_words) {
    const int off = word_offset(tbl[w]);
    int n = 1;
    while (n < kTileBlocks && w + n < n_words && word_offset(tbl[w + n]) == off) ++n;
    return {n, off};
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              int *d_status) {
    for (uint32_t i = 0; i < kWaitPolls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255) == 255 && *abort_flag) return false;
    }
    *abort_flag = 1;
    set_status(d_status, LAZY_DSTATUS_TIMEOUT);
    return false;
}

__device__ __forceinline__ void rot_sync() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// Same decision for every lane of the warp (a lane whose poll ran out aborts all).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *d_status) {
    const bool ok = wait_or_abort(bar, parity, abort_flag, d_status);
    return __all_sync(0xffffffffu, ok);
}

// Same decision for the 128 threads of the rotation warpgroup (named barrier 2).
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

template <bool PLAIN>
__global__ void __launch_bounds__(kThreads, 1) prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = align1024(smem_raw);
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kOffBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);
    float2 *segcs = reinterpret_cast<float2 *>(sm + kOffSeg);
    double *theta_s = reinterpret_cast<double *>(sm + kOffTheta);

    const int mt = blockIdx.x, kvh = blockIdx.y, r = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    const int q0 = p.cu_q[r];
    const int T = p.cu_q[r + 1] - q0;
    const int R0 = mt * kRows;
    if (R0 >= T * G) return;   // uniform: this tile has no rows
    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    const uint32_t *tbl = p.table + wbase;
    const int pos0 = p.q_pos0[r];
    const int tok_base = R0 / G;
    const int Pbase = pos0 + tok_base;

    if (threadIdx.x == 0) {
        mbar_init(&bars[B_KFULL], 1);
        mbar_init(&bars[B_KFULL + 1], 1);
        mbar_init(&bars[B_KEMPTY], 1);
        mbar_init(&bars[B_KEMPTY + 1], 1);
        mbar_init(&bars[B_VFULL], 1);
        mbar_init(&bars[B_VFULL + 1], 1);
        mbar_init(&bars[B_VEMPTY], 1);
        mbar_init(&bars[B_VEMPTY + 1], 1);
        mbar_init(&bars[B_SFULL], 1);
        mbar_init(&bars[B_SFULL + 1], 1);
        mbar_init(&bars[B_SFREE], 4);
        mbar_init(&bars[B_SFREE + 1], 4);
        mbar_init(&bars[B_PFULL], 4);
        mbar_init(&bars[B_PFULL + 1], 4);
        mbar_init(&bars[B_ODONE], 1);
        mbar_init(&bars[B_ODONE + 1], 1);
        mbar_init(&bars[B_QFULL], 4);
        mbar_init(&bars[B_QFULL + 1], 4);
        mbar_init(&bars[B_QEMPTY], 1);
        mbar_init(&bars[B_QEMPTY + 1], 1);
        mbar_init(&bars[B_DRAIN], 1);
        *abort_flag = 0;
        if (mt == 0 && kvh == 0 && n_words > p.max_words) set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (threadIdx.x < kHalfDim) theta_s[threadIdx.x] = p.rope.theta[threadIdx.x];
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tbase = *tmem_slot;
    const uint32_t tS0 = tbase, tO = tbase + 256, tP0 = tbase + 384;

    if (warp == 0) {
        // ============================================================ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int w = 0, j = 0; w < n_words; ++j) {
                const KTile t = ktile(tbl, w, n_words);
                const int st = j & 1;
                const uint32_t ph = ((j >> 1) & 1) ^ 1;
                if (!wait_or_abort(&bars[B_KEMPTY + st], ph, abort_flag, p.d_status)) break;
                mbar_arrive_expect_tx(&bars[B_KFULL + st], t.n * kBlockBytes);
                uint8_t *kd = sm + kOffK + st * kTileBytes;
                for (int k = 0; k < t.n; ++k) {
                    const uint32_t b = word_block(tbl[w + k]);
                    int row;
                    if (b >= static_cast<uint32_t>(p.num_blocks)) {
                        set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
                        row = p.k_rows;   // fully out of bounds: the box is zero-filled
                    } else {
                        row = PLAIN ? ((wbase + w + k) * p.hkv + kvh) * kBlockTokens
                                    : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                    }
                    tma_load_2d(kd + k * kBoxBytes, &tmK, 0, row, &bars[B_KFULL + st]);
                    tma_load_2d(kd + kHalfPlane + k * kBoxBytes, &tmK, kHalfDim, row, &bars[B_KFULL + st]);
                }
                if (!wait_or_abort(&bars[B_VEMPTY + st], ph, abort_flag, p.d_status)) {
                    issued = j + 1;   // K of this tile is in flight
                    break;
                }
                mbar_arrive_expect_tx(&bars[B_VFULL + st], t.n * kBlockBytes);
                uint8_t *vd = sm + kOffV + st * kTileBytes;
                for (int k = 0; k < t.n; ++k) {
                    const uint32_t b = word_block(tbl[w + k]);
                    const int row = b >= static_cast<uint32_t>(p.num_blocks)
                                        ? p.v_rows
                                        : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                    tma_load_2d(vd + k * kBoxBytes, &tmV, 0, row, &bars[B_VFULL + st]);
                    tma_load_2d(vd + kHalfPlane + k * kBoxBytes, &tmV, kHalfDim, row, &bars[B_VFULL + st]);
                }
                issued = j + 1;
                w += t.n;
            }
            // no copy may land after the CTA exits: wait for the last phase of each armed stage
            for (int j = max(0, issued - 2); j < issued; ++j) {
                mbar_wait(&bars[B_KFULL + (j & 1)], (j >> 1) & 1);
                mbar_wait(&bars[B_VFULL + (j & 1)], (j >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ============================================================ MMA issuer
        if (lane == 0) {
            const uint32_t idq = tc::idesc_bf16(128, 128, false);
            const uint32_t idv = tc::idesc_bf16(128, 128, true);
            const uint32_t sQ = smem_u32(sm + kOffQ), sK = smem_u32(sm + kOffK), sV = smem_u32(sm + kOffV);
            int seg = -1, cur = INT_MIN, prev_n = 0, j = 0;
            bool ok = true;
            auto issue_pv = [&](int t, int n) -> bool {
                const int s = t & 1;
                if (!wait_or_abort(&bars[B_VFULL + s], (t >> 1) & 1, abort_flag, p.d_status)) return false;
                if (!wait_or_abort(&bars[B_PFULL + s], (t >> 1) & 1, abort_flag, p.d_status)) return false;
                tc::fence_after_sync();
                const uint32_t vb = sV + s * kTileBytes;
                for (int k = 0; k < n; ++k)
                    tc::mma_ts(tO, tP0 + 64 * s + 8 * k, tc::smem_desc(vb + k * kBoxBytes, kHalfPlane, 1024), idv,
                               (t > 0 || k > 0) ? 1u : 0u);
                tc::commit(&bars[B_ODONE + s]);
                tc::commit(&bars[B_VEMPTY + s]);
                return true;
            };
            for (int w = 0; w < n_words && ok; ++j) {
                const KTile t = ktile(tbl, w, n_words);
                const int off_rot = PLAIN ? 0 : t.off;
                if (off_rot != cur) {
                    ++seg;
                    cur = off_rot;
                    if (!wait_or_abort(&bars[B_QFULL + (seg & 1)], (seg >> 1) & 1, abort_flag, p.d_status)) break;
                }
                const int s = j & 1;
                if (!wait_or_abort(&bars[B_KFULL + s], (j >> 1) & 1, abort_flag, p.d_status)) break;
                if (j >= 2 && !wait_or_abort(&bars[B_SFREE + s], ((j - 2) >> 1) & 1, abort_flag, p.d_status)) break;
                tc::fence_after_sync();
                const uint32_t qa = sQ + (seg & 1) * kTileBytes, kb = sK + s * kTileBytes;
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t o = (kk >> 2) * kHalfPlane + (kk & 3) * 32;
                    tc::mma_ss(tS0 + 128 * s, tc::smem_desc(qa + o, 16, 1024), tc::smem_desc(kb + o, 16, 1024), idq,
                               kk > 0 ? 1u : 0u);
                }
                tc::commit(&bars[B_SFULL + s]);
                tc::commit(&bars[B_KEMPTY + s]);
                const int wn = w + t.n;
                const bool seg_end = wn >= n_words || (PLAIN ? false : word_offset(tbl[wn]) != off_rot);
                if (seg_end) tc::commit(&bars[B_QEMPTY + (seg & 1)]);
                if (j >= 1) ok = issue_pv(j - 1, prev_n);
                prev_n = t.n;
                w = wn;
            }
            if (ok && j >= 1 && !*abort_flag) issue_pv(j - 1, prev_n);
            // every MMA this thread issued has completed before tensor memory is freed
            tc::commit(&bars[B_DRAIN]);
            mbar_wait(&bars[B_DRAIN], 0);
        }
    } else if (warp >= 4 && warp < 8) {
        // ============================================================ softmax (one row per thread)
        const int row = threadIdx.x - 128;
        const int R = R0 + row;
        const bool row_ok = R < T * G;
        const int tok = row_ok ? R / G : tok_base;
        const int g = R % G;
        const int prow = pos0 + tok;
        const uint32_t lane_off = static_cast<uint32_t>(32 * (warp - 4)) << 16;
        float m_run = -INFINITY, l_run = 0.f;
        int j = 0;
        bool ok = true;
        for (int w = 0; w < n_words; ++j) {
            const KTile t = ktile(tbl, w, n_words);
            const int s = j & 1;
            if (!warp_wait(&bars[B_SFULL + s], (j >> 1) & 1, abort_flag, p.d_status)) { ok = false; break; }
            tc::fence_after_sync();
            // block metadata of the tile (positions for the causal mask, valid slots)
            int kj0[kTileBlocks], knv[kTileBlocks];
            bool full = t.n == kTileBlocks;
#pragma unroll
            for (int k = 0; k < kTileBlocks; ++k) {
                kj0[k] = 0;
                knv[k] = 0;
                if (k < t.n) {
                    const uint32_t b = word_block(tbl[w + k]);
                    if (b < static_cast<uint32_t>(p.num_blocks)) {
                        const uint32_t mm = p.blk_meta[b];
                        kj0[k] = meta_j0(mm);
                        knv[k] = meta_valid(mm);
                    }
                }
                full = full && knv[k] == kBlockTokens && t.off + kj0[k] + kBlockTokens - 1 <= Pbase;
            }
            // pass 1 over the S row in tensor memory: masked row maximum
            float tmax = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t x[32];
                tc::ld32(tS0 + 128 * s + lane_off + 32 * c, x);
                tc::wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int col = 32 * c + e, k = col >> 4, si = col & 15;
                    const bool vis = full || (si < knv[k] && t.off + kj0[k] + si <= prow);
                    tmax = vis ? fmaxf(tmax, __uint_as_float(x[e])) : tmax;
                }
            }
            const float m_new = fmaxf(m_run, tmax);
            const bool need = m_new > m_run + kRescaleThreshold;
            float scale = 1.f;
            if (need) {
                scale = fast_exp2(m_run - m_new);
                m_run = m_new;
                l_run *= scale;
            }
            if (j > 0 && __any_sync(0xffffffffu, need)) {
                // O must be complete up to tile j-1 before it is rescaled in place
                if (!warp_wait(&bars[B_ODONE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort_flag, p.d_status)) {
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
                tc::wait_st();
            }
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            // P[j%2] is free once the PV product of tile j-2 has completed
            if (j >= 2 && !warp_wait(&bars[B_ODONE + s], ((j - 2) >> 1) & 1, abort_flag, p.d_status)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            // pass 2: P = 2^(S - m) as bf16 pairs into tensor memory, row sum in fp32
            float lsum = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t x[32], pk[16];
                tc::ld32(tS0 + 128 * s + lane_off + 32 * c, x);
                tc::wait_ld();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float pr[2];
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int col = 32 * c + 2 * e + h, k = col >> 4, si = col & 15;
                        const bool vis = full || (si < knv[k] && t.off + kj0[k] + si <= prow);
                        pr[h] = vis ? fast_exp2(__uint_as_float(x[2 * e + h]) - mu) : 0.f;
                    }
                    lsum += pr[0] + pr[1];
                    pk[e] = pack_bf16(pr[0], pr[1]);
                }
                tc::st16(tP0 + 64 * s + lane_off + 16 * c, pk);
            }
            l_run += lsum;
            tc::wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_SFREE + s]);
                mbar_arrive(&bars[B_PFULL + s]);
            }
            w += t.n;
        }
        // ------------------------------------------------------------ epilogue
        uint32_t ob[4][32];
        bool have = ok && j > 0;
        if (have) {
            have = warp_wait(&bars[B_ODONE + ((j - 1) & 1)], ((j - 1) >> 1) & 1, abort_flag, p.d_status);
        }
        const float inv = (have && l_run > 0.f) ? 1.f / l_run : 0.f;
        if (__all_sync(0xffffffffu, have)) {
            tc::fence_after_sync();
#pragma unroll
            for (int c = 0; c < 4; ++c) tc::ld32(tO + lane_off + 32 * c, ob[c]);
            tc::wait_ld();
        } else {
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) ob[c][e] = 0u;
        }
        if (row_ok) {
            uint4 *o = reinterpret_cast<uint4 *>(p.out + (static_cast<size_t>(q0 + tok) * p.hq + kvh * G + g) *
                                                             kHeadDim);
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 u;
                    u.x = pack_bf16(__uint_as_float(ob[c][8 * v + 0]) * inv, __uint_as_float(ob[c][8 * v + 1]) * inv);
                    u.y = pack_bf16(__uint_as_float(ob[c][8 * v + 2]) * inv, __uint_as_float(ob[c][8 * v + 3]) * inv);
                    u.z = pack_bf16(__uint_as_float(ob[c][8 * v + 4]) * inv, __uint_as_float(ob[c][8 * v + 5]) * inv);
                    u.w = pack_bf16(__uint_as_float(ob[c][8 * v + 6]) * inv, __uint_as_float(ob[c][8 * v + 7]) * inv);
                    o[4 * c + v] = u;
                }
        }
    } else if (warp >= 8) {
        // ============================================================ query rotation
        const int tid = threadIdx.x - 256;
        const int ch = tid & 7;          // 8-pair chunk: pairs 8ch .. 8ch+7
        const int rbase = tid >> 3;      // rows rbase + 16k
        uint8_t *qt = sm + kOffQt;
        // Qt = R(p_i - P) q_i, pre-scaled by softmax_scale * log2(e)
#pragma unroll 1
        for (int k = 0; k < 8; ++k) {
            const int rr = rbase + 16 * k;
            const int Rr = R0 + rr;
            uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
            if (Rr < T * G) {
                const int tk = Rr / G, gg = Rr % G;
                const uint16_t *q = p.q_raw + (static_cast<size_t>(q0 + tk) * p.hq + kvh * G + gg) * kHeadDim;
                const uint4 a4 = *reinterpret_cast<const uint4 *>(q + 8 * ch);
                const uint4 b4 = *reinterpret_cast<const uint4 *>(q + kHalfDim + 8 * ch);
                const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4);
                const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4);
                uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
                uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float c0, s0, c1, s1;
                    rope_cos_sin(tk - tok_base, theta_s[8 * ch + 2 * e], c0, s0);
                    rope_cos_sin(tk - tok_base, theta_s[8 * ch + 2 * e + 1], c1, s1);
                    const float a0 = bf16_lo(aw[e]) * p.scale_log2, a1 = bf16_hi(aw[e]) * p.scale_log2;
                    const float b0 = bf16_lo(bw[e]) * p.scale_log2, b1 = bf16_hi(bw[e]) * p.scale_log2;
                    lw[e] = pack_bf16(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
                    hw[e] = pack_bf16(b0 * c0 + a0 * s0, b1 * c1 + a1 * s1);
                }
            }
            const uint32_t off = rr * 128 + ((ch ^ (rr & 7)) << 4);
            *reinterpret_cast<uint4 *>(qt + off) = lo;
            *reinterpret_cast<uint4 *>(qt + kHalfPlane + off) = hi;
        }
        rot_sync();
        int seg = -1, cur = INT_MIN;
        for (int w = 0; w < n_words;) {
            const KTile t = ktile(tbl, w, n_words);
            w += t.n;
            const int off_rot = PLAIN ? 0 : t.off;
            if (off_rot == cur) continue;
            ++seg;
            cur = off_rot;
            const int qb = seg & 1;
            bool ok = true;
            if (seg >= 2) ok = wait_or_abort(&bars[B_QEMPTY + qb], ((seg - 2) >> 1) & 1, abort_flag, p.d_status);
            if (!rot_all(ok)) break;
            // the segment's uniform rotation R(P - o), one pair per thread
            if (tid < kHalfDim) {
                float c, s;
                rope_cos_sin(Pbase - off_rot, theta_s[tid], c, s);
                segcs[tid] = make_float2(c, s);
            }
            rot_sync();
            float cs[8], sn[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float2 v = segcs[8 * ch + e];
                cs[e] = v.x;
                sn[e] = v.y;
            }
            uint8_t *qd = sm + kOffQ + qb * kTileBytes;
#pragma unroll 2
            for (int k = 0; k < 8; ++k) {
                const int rr = rbase + 16 * k;
                const uint32_t off = rr * 128 + ((ch ^ (rr & 7)) << 4);
                const uint4 a4 = *reinterpret_cast<const uint4 *>(qt + off);
                const uint4 b4 = *reinterpret_cast<const uint4 *>(qt + kHalfPlane + off);
                const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4);
                const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4);
                uint4 lo, hi;
                uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
                uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a0 = bf16_lo(aw[e]), a1 = bf16_hi(aw[e]);
                    const float b0 = bf16_lo(bw[e]), b1 = bf16_hi(bw[e]);
                    const float c0 = cs[2 * e], s0 = sn[2 * e], c1 = cs[2 * e + 1], s1 = sn[2 * e + 1];
                    lw[e] = pack_bf16(a0 * c0 - b0 * s0, a1 * c1 - b1 * s1);
                    hw[e] = pack_bf16(b0 * c0 + a0 * s0, b1 * c1 + a1 * s1);
                }
                *reinterpret_cast<uint4 *>(qd + off) = lo;
                *reinterpret_cast<uint4 *>(qd + kHalfPlane + off) = hi;
            }
            fence_proxy_async_smem();   // generic-proxy writes become visible to the tensor core
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_QFULL + qb]);
            rot_sync();                 // segcs is rewritten for the next segment only after all reads
        }
    }

    // ================================================================ teardown
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tbase, 512);
    }
}

template <bool PLAIN>
cudaError_t launch_t(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, cudaStream_t s) {
    auto kern = prefill_tc_kernel<PLAIN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kTcSmem);
    if (e != cudaSuccess) return e;
    const int mtiles = (p.max_q * p.group + kRows - 1) / kRows;
    dim3 grid(max(1, mtiles), p.hkv, p.num_req);
    kern<<<grid, kThreads, kTcSmem, s>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill_tc(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, bool plain,
                              cudaStream_t s) {
    return plain ? launch_t<true>(tk, tv, p, s) : launch_t<false>(tk, tv, p, s);
}

}  // namespace lazy
