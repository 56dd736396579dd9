// prefill_mma.cu -- causal prefill attention over the paged pool with deferred
// RoPE, on warp-level tensor-core MMAs (m16n8k16).
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Prefilling -- cached KV blocks are loaded and one relative
// rotation (query position minus document offset) replaces resetting the
// keys to position 0 and rotating them again.
//
// Here the single relative rotation is applied to the query tile: for each
// segment (document) met in the table walk, every query row i of the tile is
// rotated by (p_i - o) once, and the stored keys (rotated at their local
// index j) go from HBM to the tensor cores untouched.  Scores then carry the
// angle (p_i - o - j) of eager RoPE attention.
//
// Work decomposition.  One CTA per (128-row query tile, KV head, request).
// Rows are (token, head-in-group) pairs, token-major, so one K/V block loaded
// by TMA serves all G query heads of its KV head.  Warp 8 is the TMA
// producer (one 16-token K block and V block per stage); warps 0-7 own 16
// rows each and run S = Q K^T, the online softmax and O += P V.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace lazy {

namespace {

constexpr int kPfStages = 8;
constexpr int kPfStageBytes = 2 * kBlockBytes;
constexpr int kPfRows = 128;
constexpr int kPfConsumers = 8;
constexpr int kPfThreads = (kPfConsumers + 1) * 32;
constexpr int kQTileBytes = kPfRows * kHeadDim * 2;   // 32 KiB, two swizzled halves of 128 rows
constexpr size_t kPfSmem = kPfStages * kPfStageBytes + kQTileBytes + 1024;

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}
__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kPfConsumers * 32) : "memory");
}

template <bool PLAIN>
__global__ void __launch_bounds__(kPfThreads) prefill_mma_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                 const __grid_constant__ CUtensorMap tmV,
                                                                 const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align1024(smem_raw);
    uint8_t *qtile = stages + kPfStages * kPfStageBytes;
    __shared__ uint64_t full_bar[kPfStages], empty_bar[kPfStages];
    __shared__ double theta_s[kHalfDim];

    const int mt = blockIdx.x, kvh = blockIdx.y, r = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;
    const int q0 = p.cu_q[r];
    const int T = p.cu_q[r + 1] - q0;
    const int R0 = mt * kPfRows;
    if (R0 >= T * G) return;   // whole CTA beyond this request's rows (uniform exit)
    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    const int pos0 = p.q_pos0[r];

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPfStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kPfConsumers);
        }
        if (mt == 0 && kvh == 0 && n_words > p.max_words) set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (threadIdx.x < kHalfDim) theta_s[threadIdx.x] = p.rope.theta[threadIdx.x];
    __syncthreads();

    if (warp == kPfConsumers) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmK);
            tma_prefetch_desc(&tmV);
            int issued = 0;
            for (int i = 0; i < n_words; ++i) {
                const int st = i % kPfStages;
                const uint32_t ph = (i / kPfStages) & 1;
                if (!mbar_wait(&empty_bar[st], ph ^ 1)) {
                    set_status(p.d_status, LAZY_DSTATUS_TIMEOUT);
                    break;
                }
                const int widx = wbase + i;
                const uint32_t w = p.table[widx];
                const uint32_t b = word_block(w);
                issued = i + 1;
                if (b >= static_cast<uint32_t>(p.num_blocks)) {
                    set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
                    mbar_arrive(&full_bar[st]);
                    continue;
                }
                mbar_arrive_expect_tx(&full_bar[st], kPfStageBytes);
                uint8_t *dst = stages + st * kPfStageBytes;
                const int krow = PLAIN ? (widx * p.hkv + kvh) * kBlockTokens
                                       : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                const int vrow = (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                tma_load_block(dst, &tmK, krow, &full_bar[st]);
                tma_load_block(dst + kBlockBytes, &tmV, vrow, &full_bar[st]);
            }
            for (int i = max(0, issued - kPfStages); i < issued; ++i)
                mbar_wait(&full_bar[i % kPfStages], (i / kPfStages) & 1);
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const int c = lane & 3, rr = lane >> 2;
    // rows of this thread: R0 + 16*warp + rr and + 8
    int rowpos[2];
    bool rowok[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const int R = R0 + 16 * warp + rr + 8 * k;
        rowok[k] = R < T * G;
        rowpos[k] = pos0 + (rowok[k] ? R / G : 0);
    }
    // warp-uniform: does this warp own any real row, and the latest position among them
    const bool warp_active = R0 + 16 * warp < T * G;
    const int warp_max_pos = pos0 + min(R0 + 16 * warp + 15, T * G - 1) / G;

    float oacc[16][4];
#pragma unroll
    for (int t = 0; t < 16; ++t) oacc[t][0] = oacc[t][1] = oacc[t][2] = oacc[t][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    uint32_t qa[8][4];
    int cur_off = INT_MIN;
    const uint32_t stage0 = smem_u32(stages);
    const uint32_t qt0 = smem_u32(qtile);
    const int mi = lane >> 3, li = lane & 7;
    const int q_row = 16 * warp + li + 8 * (mi & 1), q_dc = 8 * (mi >> 1);   // Q as A (rows x d)
    const int k_key = li + 8 * (mi >> 1), k_dc = 8 * (mi & 1);               // K^T as B (non-trans)
    const int v_key = li + 8 * (mi & 1), v_dc = 8 * (mi >> 1);               // V as B (.trans)
    const int tok_lo = R0 / G, tok_hi = min(T - 1, (R0 + kPfRows - 1) / G);
    // rows past the request's last token are never written; keep them zero
    for (int it = threadIdx.x; it < kQTileBytes / 16; it += kPfConsumers * 32)
        reinterpret_cast<uint4 *>(qtile)[it] = make_uint4(0, 0, 0, 0);

    for (int i = 0; i < n_words; ++i) {
        const int st = i % kPfStages;
        const uint32_t ph = (i / kPfStages) & 1;
        const uint32_t w = p.table[wbase + i];
        const uint32_t b = word_block(w);
        const int off = word_offset(w);
        const int off_rot = PLAIN ? 0 : off;
        if (b < static_cast<uint32_t>(p.num_blocks) && off_rot != cur_off) {
            // one relative rotation of the whole query tile for this segment
            cur_off = off_rot;
            consumer_sync();   // everyone has loaded fragments of the previous rotation
            const int ntok = tok_hi - tok_lo + 1;
            for (int it = threadIdx.x; it < ntok * kHalfDim; it += kPfConsumers * 32) {
                const int tl = it / kHalfDim, ip = it % kHalfDim;
                const int tok = tok_lo + tl;
                float cs, sn;
                rope_cos_sin(pos0 + tok - off_rot, theta_s[ip], cs, sn);
                for (int g = 0; g < G; ++g) {
                    const int row = tok * G + g - R0;
                    if (row < 0 || row >= kPfRows) continue;
                    const uint16_t *q = p.q_raw + (static_cast<size_t>(q0 + tok) * p.hq + kvh * G + g) * kHeadDim;
                    const float a = bits_to_float(q[ip]) * p.scale_log2;
                    const float bq = bits_to_float(q[ip + kHalfDim]) * p.scale_log2;
                    __nv_bfloat16 ra = __float2bfloat16_rn(a * cs - bq * sn);
                    __nv_bfloat16 rb = __float2bfloat16_rn(bq * cs + a * sn);
                    *reinterpret_cast<__nv_bfloat16 *>(qtile + swz_offset(row, ip, kPfRows)) = ra;
                    *reinterpret_cast<__nv_bfloat16 *>(qtile + swz_offset(row, ip + kHalfDim, kPfRows)) = rb;
                }
            }
            // rows beyond the request stay as whatever is there; they are never written out
            consumer_sync();
#pragma unroll
            for (int s = 0; s < 8; ++s)
                ldsm_x4(qt0 + swz_offset(q_row, 16 * s + q_dc, kPfRows), qa[s][0], qa[s][1], qa[s][2], qa[s][3]);
        }
        if (!mbar_wait(&full_bar[st], ph)) {
            set_status(p.d_status, LAZY_DSTATUS_TIMEOUT);
            break;
        }
        if (b < static_cast<uint32_t>(p.num_blocks)) {
            const uint32_t meta = p.blk_meta[b];
            const int j0 = meta_j0(meta), nv = meta_valid(meta);
            const int kpos0 = off + j0;
            const uint32_t kbase = stage0 + st * kPfStageBytes;
            const uint32_t vbase = kbase + kBlockBytes;
            if (warp_active && kpos0 <= warp_max_pos) {
                float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(kbase + swz_offset(k_key, 16 * s + k_dc, kBlockTokens), b0, b1, b2, b3);
                    mma_bf16(sacc[0], qa[s][0], qa[s][1], qa[s][2], qa[s][3], b0, b1);
                    mma_bf16(sacc[1], qa[s][0], qa[s][1], qa[s][2], qa[s][3], b2, b3);
                }
                // mask: key 8n + 2c + e visible to row k iff valid slot and kpos <= rowpos
                const bool full_vis = nv == kBlockTokens && kpos0 + kBlockTokens - 1 <= min(rowpos[0], rowpos[1]);
                if (!full_vis) {
#pragma unroll
                    for (int n = 0; n < 2; ++n)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int key = 8 * n + 2 * c + (e & 1);
                            const int k = e >> 1;
                            if (!(key < nv && kpos0 + key <= rowpos[k])) sacc[n][e] = -INFINITY;
                        }
                }
                float pr[2][4];
#pragma unroll
                for (int k = 0; k < 2; ++k) {
                    float bm = fmaxf(fmaxf(sacc[0][2 * k], sacc[0][2 * k + 1]), fmaxf(sacc[1][2 * k], sacc[1][2 * k + 1]));
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 1));
                    bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, 2));
                    const float mn = fmaxf(m_run[k], bm);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    const float sc = fast_exp2(m_run[k] - mu);
                    if (sc != 1.f) {
                        l_run[k] *= sc;
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            oacc[t][2 * k] *= sc;
                            oacc[t][2 * k + 1] *= sc;
                        }
                    }
                    m_run[k] = mn;
#pragma unroll
                    for (int n = 0; n < 2; ++n) {
                        pr[n][2 * k] = fast_exp2(sacc[n][2 * k] - mu);
                        pr[n][2 * k + 1] = fast_exp2(sacc[n][2 * k + 1] - mu);
                        l_run[k] += pr[n][2 * k] + pr[n][2 * k + 1];
                    }
                }
                const uint32_t a0 = pack_bf16(pr[0][0], pr[0][1]);
                const uint32_t a1 = pack_bf16(pr[0][2], pr[0][3]);
                const uint32_t a2 = pack_bf16(pr[1][0], pr[1][1]);
                const uint32_t a3 = pack_bf16(pr[1][2], pr[1][3]);
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(vbase + swz_offset(v_key, 16 * t + v_dc, kBlockTokens), b0, b1, b2, b3);
                    mma_bf16(oacc[2 * t], a0, a1, a2, a3, b0, b1);
                    mma_bf16(oacc[2 * t + 1], a0, a1, a2, a3, b2, b3);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[st]);
    }

    // ---------------------------------------------------------------- epilogue
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        l_run[k] += __shfl_xor_sync(0xffffffffu, l_run[k], 1);
        l_run[k] += __shfl_xor_sync(0xffffffffu, l_run[k], 2);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        if (!rowok[k]) continue;
        const int R = R0 + 16 * warp + rr + 8 * k;
        const int tok = R / G, g = R % G;
        uint16_t *o = p.out + (static_cast<size_t>(q0 + tok) * p.hq + kvh * G + g) * kHeadDim;
        const float inv = l_run[k] > 0.f ? 1.f / l_run[k] : 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t)
            *reinterpret_cast<uint32_t *>(o + 8 * t + 2 * c) = pack_bf16(oacc[t][2 * k] * inv, oacc[t][2 * k + 1] * inv);
    }
}

template <bool PLAIN>
cudaError_t launch_prefill_t(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, cudaStream_t s) {
    auto kern = prefill_mma_kernel<PLAIN>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPfSmem);
    if (e != cudaSuccess) return e;
    const int mtiles = (p.max_q * p.group + kPfRows - 1) / kPfRows;
    dim3 grid(max(1, mtiles), p.hkv, p.num_req);
    kern<<<grid, kPfThreads, kPfSmem, s>>>(tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, bool plain,
                           cudaStream_t s) {
    return plain ? launch_prefill_t<true>(tk, tv, p, s) : launch_prefill_t<false>(tk, tv, p, s);
}

}  // namespace lazy
