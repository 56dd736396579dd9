// decode.cu -- split-K decode attention over the paged pool with deferred RoPE.
//
// Source: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary, Technical
// Implementation: Decoding -- one query token per request (M = 1); the
// rotation lives inside the inner loop, and the query is rotated again just
// at a change of segment offset (a new document); the (block ID, offset)
// metadata is decoded from one register; the kernel reads only K and V.
//
// Work decomposition (G <= 8 query heads per KV head; more heads run on the
// tensor-memory kernel of decode_tc.cu).  One CTA per (split, KV head,
// request); a split is a range of consecutive table words (16-token blocks).
// Warp 4 is the TMA producer: for each word it loads the K block and the V
// block (4 KiB each, two 128-byte-swizzled boxes) into a ring of shared-memory
// stages.  Warps 0-3 consume: the G query heads of the KV head form the N
// dimension of m16n8k16 tensor-core MMAs (S^T = K q^T, then O^T += V^T P^T),
// so each K/V byte is read from HBM once and feeds all G heads.  Warps split
// the words of a stage ring round-robin.  Per-warp online-softmax states are
// merged in shared memory; split partials (m, l, acc) go to the workspace and
// a second kernel combines them (flash-decoding).
//
// ALiBi (p.alibi): the frequency table is zero, so the query "rotation" is the
// identity and runs once; each score gets slope_h * (o + j - p) in log2 units,
// with o + j from the table word and the block's local index, as the mask uses.
#include <climits>

#include "common.cuh"
#include "kernels.h"

namespace lazy {

namespace {

constexpr int kStageBytes = 2 * kBlockBytes;     // K + V of one word
constexpr int kDecodeThreads = 160;               // 4 consumer warps + 1 producer warp
constexpr int kDefaultStages = 8;
__host__ __device__ constexpr size_t decode_smem(int stages) { return size_t(stages) * kStageBytes + 1024; }

__device__ __forceinline__ uint8_t *align1024(uint8_t *p) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Producer warp of the decode kernels.  The warp fetches the split's table words and their
// blocks' metadata 32 at a time, one word per lane (two dependent global loads per 32 words
// instead of per word); lane 0 then arms the stages in word order with the values shuffled to
// it: each stage gets the word's K block and V block (4 KiB each) by TMA, and the word and the
// block's metadata travel with the stage in shared memory.
template <bool PLAIN, int kDecodeStages>
__device__ __forceinline__ void decode_producer(const CUtensorMap &tmK, const CUtensorMap &tmV, const AttnParams &p,
                                                uint8_t *stages, uint64_t *full_bar, uint64_t *empty_bar,
                                                uint32_t *stage_word, uint32_t *stage_meta, int kvh, int wbase,
                                                int lo, int cnt, int lane) {
    if (lane == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    int issued = 0;
    bool stop = false;
    for (int i0 = 0; i0 < cnt && !stop; i0 += 32) {
        uint32_t w_l = 0u, m_l = 0u;
        if (i0 + lane < cnt) {
            w_l = p.table[wbase + lo + i0 + lane];
            const uint32_t b = word_block(w_l);
            if (b < static_cast<uint32_t>(p.num_blocks)) m_l = p.blk_meta[b];
        }
        const int n = min(32, cnt - i0);
        for (int k = 0; k < n; ++k) {
            const uint32_t w = __shfl_sync(0xffffffffu, w_l, k);
            const uint32_t meta = __shfl_sync(0xffffffffu, m_l, k);
            if (lane == 0) {
                const int i = i0 + k;
                const int st = i % kDecodeStages;
                const uint32_t ph = (i / kDecodeStages) & 1;
                if (!mbar_wait(&empty_bar[st], ph ^ 1)) {
                    set_status(p.d_status, LAZY_DSTATUS_TIMEOUT);
                    stop = true;
                } else {
                    const int widx = wbase + lo + i;
                    const uint32_t b = word_block(w);
                    issued = i + 1;
                    stage_word[st] = w;
                    if (b >= static_cast<uint32_t>(p.num_blocks)) {
                        stage_meta[st] = 0u;
                        set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
                        mbar_arrive(&full_bar[st]);   // completes the phase with no data
                    } else {
                        stage_meta[st] = meta;
                        mbar_arrive_expect_tx(&full_bar[st], kStageBytes);
                        uint8_t *dst = stages + st * kStageBytes;
                        const int krow = PLAIN ? (widx * p.hkv + kvh) * kBlockTokens
                                               : (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                        const int vrow = (static_cast<int>(b) * p.hkv + kvh) * kBlockTokens;
                        tma_load_block(dst, &tmK, krow, &full_bar[st]);
                        tma_load_block(dst + kBlockBytes, &tmV, vrow, &full_bar[st]);
                    }
                }
            }
            if (__shfl_sync(0xffffffffu, stop ? 1 : 0, 0)) {
                stop = true;
                break;
            }
        }
    }
    if (lane == 0) {
        // Never leave with copies in flight: wait for the last phase of
        // every stage this thread armed (immediate on the normal path).
        for (int i = max(0, issued - kDecodeStages); i < issued; ++i)
            mbar_wait(&full_bar[i % kDecodeStages], (i / kDecodeStages) & 1);
    }
}

// NT: groups of 8 query heads per KV head (1 for G <= 8, 2 for G <= 16, 4 for G <= 32).
// PLAIN: keys come from a materialised copy indexed by table position, and the
// query is rotated once at its absolute position (the comparison path).
// Stage i of the ring holds word i mod kDecodeStages, and consumer warp kl takes
// words i = kl (mod KW).  The ring size is a multiple of KW, so a stage always
// returns to the same warp: a warp's parity wait on a stage can then never
// run ahead of that stage's previous round (which another warp would own).
template <int NT, bool PLAIN, int kDecodeStages>
__global__ void __launch_bounds__(kDecodeThreads, 3) decode_split_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                      const __grid_constant__ CUtensorMap tmV,
                                                                      const AttnParams p) {
    constexpr int KW = 4 / NT;   // warps sharing the words of one head group
    static_assert(kDecodeStages % 4 == 0, "the stage ring must be a multiple of the consumer warps");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *stages = align1024(smem_raw);
    __shared__ uint64_t full_bar[kDecodeStages], empty_bar[kDecodeStages];
    __shared__ uint32_t stage_word[kDecodeStages], stage_meta[kDecodeStages];
    __shared__ double theta_s[kHalfDim];
    __shared__ float slope_s[32];   // ALiBi slope (log2 units) of head g of the group; 0 past G

    const int split = blockIdx.x, kvh = blockIdx.y, r = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = p.group;

    const int wbase = p.table_indptr[r];
    const int n_words = p.table_indptr[r + 1] - wbase;
    const int lo = split * p.words_per_split;
    const int cnt = max(0, min(n_words, lo + p.words_per_split) - lo);
    const int qpos = p.q_pos[r];

    if (threadIdx.x == 0) {
        for (int s = 0; s < kDecodeStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NT);
        }
        if (split == 0 && n_words > p.max_words) set_status(p.d_status, LAZY_DSTATUS_BAD_TABLE);
        fence_barrier_init();
    }
    if (threadIdx.x < kHalfDim) theta_s[threadIdx.x] = p.rope.theta[threadIdx.x];
    if (threadIdx.x < 32) slope_s[threadIdx.x] = (p.alibi && threadIdx.x < G) ? p.alibi_log2[kvh * G + threadIdx.x] : 0.f;
    __syncthreads();

    // per-thread softmax state for query heads (8*ht + 2c, 8*ht + 2c + 1)
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float oacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
    const int ht = warp % NT, kl = warp / NT;
    const int c = lane & 3, rr = lane >> 2;

    if (warp == 4) {
        decode_producer<PLAIN, kDecodeStages>(tmK, tmV, p, stages, full_bar, empty_bar, stage_word, stage_meta,
                                              kvh, wbase, lo, cnt, lane);
    } else {
        // ------------------------------------------------------------ consumers
        // raw query of head g = 8*ht + rr in B-fragment order, pre-scaled
        const int g_b = 8 * ht + rr;
        float qf[8][4];
        {
            const uint16_t *q = p.q_raw + (static_cast<size_t>(r) * p.hq + kvh * G + g_b) * kHeadDim;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
                const int d0 = 16 * s + 2 * c;
                if (g_b < G) {
                    const uint32_t w0 = *reinterpret_cast<const uint32_t *>(q + d0);
                    const uint32_t w1 = *reinterpret_cast<const uint32_t *>(q + d0 + 8);
                    qf[s][0] = bf16_lo(w0) * p.scale_log2;
                    qf[s][1] = bf16_hi(w0) * p.scale_log2;
                    qf[s][2] = bf16_lo(w1) * p.scale_log2;
                    qf[s][3] = bf16_hi(w1) * p.scale_log2;
                } else {
                    qf[s][0] = qf[s][1] = qf[s][2] = qf[s][3] = 0.f;
                }
            }
        }
        uint32_t qb[8][2];
        int cur_off = INT_MIN;
        // ALiBi slopes of this thread's two score columns (heads 8*ht + 2c, 8*ht + 2c + 1)
        const float sl0 = slope_s[8 * ht + 2 * c], sl1 = slope_s[8 * ht + 2 * c + 1];
        const uint32_t stage0 = smem_u32(stages);
        // ldmatrix lane roles
        const int mi = lane >> 3, li = lane & 7;
        const int k_key = li + 8 * (mi & 1), k_dc = 8 * (mi >> 1);     // K as A operand (rows = keys)
        const int v_key = li + 8 * (mi >> 1), v_dc = 8 * (mi & 1);     // V^T as A operand via .trans

        for (int i = kl; i < cnt; i += KW) {
            const int st = i % kDecodeStages;
            const uint32_t ph = (i / kDecodeStages) & 1;
            if (!mbar_wait(&full_bar[st], ph)) {
                set_status(p.d_status, LAZY_DSTATUS_TIMEOUT);
                break;
            }
            const uint32_t w = stage_word[st];
            const uint32_t b = word_block(w);
            if (b < static_cast<uint32_t>(p.num_blocks)) {
                const uint32_t meta = stage_meta[st];
                const int off = word_offset(w);
                const int off_rot = PLAIN ? 0 : (p.alibi ? qpos : off);
                if (off_rot != cur_off) {
                    // re-rotate the query by (q_pos - offset): pairs (i, i+64)
                    // live in k-steps s and s+4 of the same thread
                    cur_off = off_rot;
                    const int delta = qpos - off_rot;
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        float ra[4], rb[4];
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            const int ip = 16 * s + 2 * c + (x & 1) + 8 * (x >> 1);
                            float cs, sn;
                            rope_cos_sin(delta, theta_s[ip], cs, sn);
                            const float a = qf[s][x], bq = qf[s + 4][x];
                            ra[x] = a * cs - bq * sn;
                            rb[x] = bq * cs + a * sn;
                        }
                        qb[s][0] = pack_bf16(ra[0], ra[1]);
                        qb[s][1] = pack_bf16(ra[2], ra[3]);
                        qb[s + 4][0] = pack_bf16(rb[0], rb[1]);
                        qb[s + 4][1] = pack_bf16(rb[2], rb[3]);
                    }
                }
                const uint32_t kbase = stage0 + st * kStageBytes;
                const uint32_t vbase = kbase + kBlockBytes;
                // S^T[16 keys][8 heads] = K q^T, the 8 k-steps in two independent chains
                float sacc[4] = {0.f, 0.f, 0.f, 0.f}, sacc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(kbase + swz_offset(k_key, 16 * s + k_dc, kBlockTokens), a0, a1, a2, a3);
                    mma_bf16((s & 1) ? sacc2 : sacc, a0, a1, a2, a3, qb[s][0], qb[s][1]);
                }
#pragma unroll
                for (int x = 0; x < 4; ++x) sacc[x] += sacc2[x];
                const int j0 = meta_j0(meta), nv = meta_valid(meta);
                if (p.alibi) {
                    // slope * (key position - query position) for keys rr and rr + 8
                    const float d0 = static_cast<float>(off + j0 + rr - qpos), d1 = d0 + 8.f;
                    sacc[0] = fmaf(sl0, d0, sacc[0]);
                    sacc[1] = fmaf(sl1, d0, sacc[1]);
                    sacc[2] = fmaf(sl0, d1, sacc[2]);
                    sacc[3] = fmaf(sl1, d1, sacc[3]);
                }
                // causal / validity mask for keys rr and rr + 8
                const bool vis0 = rr < nv && off + j0 + rr <= qpos;
                const bool vis1 = rr + 8 < nv && off + j0 + rr + 8 <= qpos;
                if (!vis0) sacc[0] = sacc[1] = -INFINITY;
                if (!vis1) sacc[2] = sacc[3] = -INFINITY;
                float bm[2] = {fmaxf(sacc[0], sacc[2]), fmaxf(sacc[1], sacc[3])};
#pragma unroll
                for (int x = 4; x < 32; x <<= 1) {
                    bm[0] = fmaxf(bm[0], __shfl_xor_sync(0xffffffffu, bm[0], x));
                    bm[1] = fmaxf(bm[1], __shfl_xor_sync(0xffffffffu, bm[1], x));
                }
                float pr[4];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float mn = fmaxf(m_run[j], bm[j]);
                    const float mu = mn == -INFINITY ? 0.f : mn;
                    // the rescale factor is exactly 1 while the running max stands (most words)
                    float sc = 1.f;
                    if (mn != m_run[j]) sc = fast_exp2(m_run[j] - mu);
                    if (sc != 1.f) {
                        l_run[j] *= sc;
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            oacc[t][j] *= sc;
                            oacc[t][j + 2] *= sc;
                        }
                    }
                    m_run[j] = mn;
                    pr[j] = fast_exp2(sacc[j] - mu);
                    pr[j + 2] = fast_exp2(sacc[j + 2] - mu);
                    l_run[j] += pr[j] + pr[j + 2];
                }
                // P^T (keys x heads) -> B fragments (keys x heads, col-major) via transpose
                const uint32_t pb0 = movmatrix_t(pack_bf16(pr[0], pr[1]));
                const uint32_t pb1 = movmatrix_t(pack_bf16(pr[2], pr[3]));
                // O^T[128 d][8 heads] += V^T P^T
#pragma unroll
                for (int t = 0; t < 8; ++t) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(vbase + swz_offset(v_key, 16 * t + v_dc, kBlockTokens), a0, a1, a2, a3);
                    mma_bf16(oacc[t], a0, a1, a2, a3, pb0, pb1);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int x = 4; x < 32; x <<= 1) l_run[j] += __shfl_xor_sync(0xffffffffu, l_run[j], x);
    }
    __syncthreads();   // every stage consumed, every copy landed: stage memory is free

    // ---------------------------------------------------------------- merge warps, write split partial
    float *sm_acc = reinterpret_cast<float *>(stages);           // [KW][8*NT][128]
    float *sm_m = sm_acc + KW * 8 * NT * kHeadDim;               // [KW][8*NT]
    float *sm_l = sm_m + KW * 8 * NT;
    if (warp < 4) {
#pragma unroll
        for (int t = 0; t < 8; ++t)
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int d = 16 * t + rr + 8 * (k >> 1);
                const int g = 8 * ht + 2 * c + (k & 1);
                sm_acc[(kl * 8 * NT + g) * kHeadDim + d] = oacc[t][k];
            }
        if (rr == 0) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                sm_m[kl * 8 * NT + 8 * ht + 2 * c + j] = m_run[j];
                sm_l[kl * 8 * NT + 8 * ht + 2 * c + j] = l_run[j];
            }
        }
    }
    __syncthreads();
    const size_t part = (static_cast<size_t>(r) * p.hkv + kvh) * p.n_splits + split;
    for (int it = threadIdx.x; it < G * kHeadDim; it += blockDim.x) {
        const int g = it / kHeadDim, d = it % kHeadDim;
        float M = -INFINITY;
#pragma unroll
        for (int k = 0; k < KW; ++k) M = fmaxf(M, sm_m[k * 8 * NT + g]);
        float L = 0.f, A = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int k = 0; k < KW; ++k) {
                const float wgt = fast_exp2(sm_m[k * 8 * NT + g] - M);
                L += wgt * sm_l[k * 8 * NT + g];
                A += wgt * sm_acc[(k * 8 * NT + g) * kHeadDim + d];
            }
        }
        p.ws_acc[(part * G + g) * kHeadDim + d] = A;
        if (d == 0) {
            p.ws_ml[(part * G + g) * 2 + 0] = M;
            p.ws_ml[(part * G + g) * 2 + 1] = L;
        }
    }
}

// out[r][h][:] = sum_s acc_s 2^(m_s - M) / sum_s l_s 2^(m_s - M); zero if nothing was visible.
__global__ void __launch_bounds__(128) decode_combine_kernel(const AttnParams p) {
    const int h = blockIdx.x % p.hq, r = blockIdx.x / p.hq;
    const int kvh = h / p.group, g = h % p.group;
    const int d = threadIdx.x;
    const size_t base = (static_cast<size_t>(r) * p.hkv + kvh) * p.n_splits;
    float M = -INFINITY;
    for (int s = 0; s < p.n_splits; ++s) M = fmaxf(M, p.ws_ml[((base + s) * p.group + g) * 2]);
    float L = 0.f, A = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < p.n_splits; ++s) {
            const size_t e = (base + s) * p.group + g;
            const float wgt = fast_exp2(p.ws_ml[e * 2] - M);
            L += wgt * p.ws_ml[e * 2 + 1];
            A += wgt * p.ws_acc[e * kHeadDim + d];
        }
    }
    const float o = L > 0.f ? A / L : 0.f;
    __nv_bfloat16 ob = __float2bfloat16_rn(o);
    p.out[(static_cast<size_t>(r) * p.hq + h) * kHeadDim + d] = *reinterpret_cast<uint16_t *>(&ob);
}

template <int NT, bool PLAIN, int NS>
cudaError_t launch_decode_t(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, cudaStream_t s) {
    auto kern = decode_split_kernel<NT, PLAIN, NS>;
    const size_t smem = decode_smem(NS);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.n_splits, p.hkv, p.num_req);
    kern<<<grid, kDecodeThreads, smem, s>>>(tk, tv, p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    decode_combine_kernel<<<p.num_req * p.hq, kHeadDim, 0, s>>>(p);
    return cudaGetLastError();
}

// Pipeline depth: kDefaultStages stages of 8 KiB per CTA (a multiple of 4).
template <int NT, bool PLAIN>
cudaError_t launch_decode_nt(const CUtensorMap &tk, const CUtensorMap &tv, const AttnParams &p, cudaStream_t s) {
    return launch_decode_t<NT, PLAIN, kDefaultStages>(tk, tv, p, s);
}

}  // namespace

DecodePlan decode_plan(int num_req, int hkv, int max_words, int group) {
    DecodePlan pl;
    const int units = max(1, num_req * hkv);
    const bool tc = group >= kDecodeTcMinGroup;
    // warp-MMA kernels: about 2000 CTAs (several waves over 148 SMs at ~3 resident CTAs each),
    // at least 8 words (128 keys) per split; tensor-memory kernel (one CTA per SM): about 600
    // CTAs, at least 16 words (two key tiles) per split
    const int target = tc ? 592 : 2048;
    const int min_words = tc ? 16 : 8;
    int splits = (target + units - 1) / units;
    const int max_splits = max(1, (max_words + min_words - 1) / min_words);
    splits = max(1, min(splits, max_splits));
    const int wps = max(1, (max_words + splits - 1) / splits);
    pl.words_per_split = wps;
    pl.grid_splits = max(1, (max_words + wps - 1) / wps);
    pl.n_splits = tc ? 2 * pl.grid_splits : pl.grid_splits;
    return pl;
}

cudaError_t launch_decode(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                          const CUtensorMap &tv8, const AttnParams &p, bool plain, cudaStream_t s) {
    // G <= 8: heads as the N dimension of warp MMAs (one warp's 8 heads share every K/V
    // fragment); more heads per KV head: heads as the rows of tcgen05 MMAs in tensor memory
    if (p.group >= kDecodeTcMinGroup) return launch_decode_tc(tk, tv, tk8, tv8, p, plain, s);
    return plain ? launch_decode_nt<1, true>(tk, tv, p, s) : launch_decode_nt<1, false>(tk, tv, p, s);
}

cudaError_t launch_decode_combine(const AttnParams &p, cudaStream_t s) {
    decode_combine_kernel<<<p.num_req * p.hq, kHeadDim, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace lazy
