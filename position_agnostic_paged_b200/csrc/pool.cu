// pool.cu -- kernels that write or copy the paged pool:
//   kv_write_kernel        keys rotated at their local index j, values copied
//   decode_table_kernel    per-slot decoding of table words (test export)
//   materialize_k_kernel   position-adjusted key copies (comparison path)
//
// Sources: gist.science, "LazyAttention: Efficient Retrieval-Augmented
// Generation with Deferred Positional Encoding", Technical Summary: Core
// Concept (deferred positional encoding) and Technical Implementation:
// Decoding (block id and offset packed in one word); shd-paper.top, same
// title, English abstract (materialisation of re-encoded copies is the cost
// the method avoids).
#include "common.cuh"
#include "kernels.h"

namespace lazy {

// One CTA per token, 128 threads.  Thread i < 64 evaluates the angle of pair
// (i, i + 64) once; the rotation is then applied to every KV head.
__global__ void __launch_bounds__(128) kv_write_kernel(KvWriteParams p) {
    const int t = blockIdx.x;
    const int tid = threadIdx.x;
    __shared__ float cs[kHalfDim], sn[kHalfDim];
    const int slot = p.slot[t];
    const int j = p.local_j[t];
    const bool bad_slot = slot < 0 || static_cast<int64_t>(slot) >= static_cast<int64_t>(p.num_blocks) * kBlockTokens;
    const bool bad_align = j < 0 || (j & (kBlockTokens - 1)) != (slot & (kBlockTokens - 1));
    if (bad_slot || bad_align) {
        if (tid == 0) set_status(p.d_status, bad_slot ? LAZY_DSTATUS_BAD_SLOT : LAZY_DSTATUS_BAD_ALIGN);
        return;
    }
    if (tid < kHalfDim) rope_cos_sin(j, p.rope.theta[tid], cs[tid], sn[tid]);
    __syncthreads();
    const int blk = slot / kBlockTokens, s = slot % kBlockTokens;
    for (int h = 0; h < p.hkv; ++h) {
        const size_t src = (static_cast<size_t>(t) * p.hkv + h) * kHeadDim;
        const size_t dst = ((static_cast<size_t>(blk) * p.hkv + h) * kBlockTokens + s) * kHeadDim;
        if (tid < kHalfDim) {
            float a = bits_to_float(p.k_raw[src + tid]);
            float b = bits_to_float(p.k_raw[src + tid + kHalfDim]);
            float c = cs[tid], sv = sn[tid];
            __nv_bfloat16 ra = __float2bfloat16_rn(a * c - b * sv);
            __nv_bfloat16 rb = __float2bfloat16_rn(b * c + a * sv);
            p.k_pool[dst + tid] = *reinterpret_cast<uint16_t *>(&ra);
            p.k_pool[dst + tid + kHalfDim] = *reinterpret_cast<uint16_t *>(&rb);
        }
        p.v_pool[dst + tid] = p.v_raw[src + tid];
    }
    if (tid == 0) atomicMax(&p.blk_meta[blk], (static_cast<uint32_t>(j / kBlockTokens) << 8) | static_cast<uint32_t>(s + 1));
}

// One thread per (word, slot).
__global__ void decode_table_kernel(DecodeTableParams p) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= p.n_words * kBlockTokens) return;
    const int64_t w = i / kBlockTokens;
    const int s = static_cast<int>(i % kBlockTokens);
    const uint32_t word = p.table[w];
    const uint32_t b = word_block(word);
    if (b >= static_cast<uint32_t>(p.num_blocks)) {
        p.out_block[i] = -1;
        p.out_slot[i] = -1;
        p.out_pos[i] = -1;
        if (s == 0) set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
        return;
    }
    const uint32_t m = p.blk_meta[b];
    p.out_block[i] = static_cast<int32_t>(b);
    p.out_slot[i] = static_cast<int32_t>(b) * kBlockTokens + s;
    p.out_pos[i] = s < meta_valid(m) ? word_offset(word) + meta_j0(m) + s : -1;
}

// One CTA per table word, 256 threads.  Each thread rotates 8 pairs (16 B
// from each half of a 256-byte key row) by the word's offset o.
__global__ void __launch_bounds__(256) materialize_k_kernel(MaterializeParams p) {
    const int w = blockIdx.x;
    const int tid = threadIdx.x;
    __shared__ float cs[kHalfDim], sn[kHalfDim];
    const uint32_t word = p.table[w];
    const uint32_t b = word_block(word);
    const bool bad = b >= static_cast<uint32_t>(p.num_blocks);
    const int nv = bad ? 0 : meta_valid(p.blk_meta[b]);
    if (bad && tid == 0) set_status(p.d_status, LAZY_DSTATUS_BAD_BLOCK);
    if (tid < kHalfDim) rope_cos_sin(word_offset(word), p.rope.theta[tid], cs[tid], sn[tid]);
    __syncthreads();
    const int items = p.hkv * kBlockTokens * 8;   // (head, slot, 8-pair chunk)
    for (int it = tid; it < items; it += blockDim.x) {
        const int chunk = it & 7;
        const int s = (it >> 3) & (kBlockTokens - 1);
        const int h = it >> 7;
        const size_t dst = ((static_cast<size_t>(w) * p.hkv + h) * kBlockTokens + s) * kHeadDim + chunk * 8;
        uint4 lo = make_uint4(0, 0, 0, 0), hi = make_uint4(0, 0, 0, 0);
        if (s < nv) {
            const size_t src = ((static_cast<size_t>(b) * p.hkv + h) * kBlockTokens + s) * kHeadDim + chunk * 8;
            const uint4 a4 = *reinterpret_cast<const uint4 *>(p.k_pool + src);
            const uint4 b4 = *reinterpret_cast<const uint4 *>(p.k_pool + src + kHalfDim);
            const uint32_t *aw = reinterpret_cast<const uint32_t *>(&a4);
            const uint32_t *bw = reinterpret_cast<const uint32_t *>(&b4);
            uint32_t *lw = reinterpret_cast<uint32_t *>(&lo);
            uint32_t *hw = reinterpret_cast<uint32_t *>(&hi);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int i0 = chunk * 8 + 2 * q, i1 = i0 + 1;
                const float a0 = bf16_lo(aw[q]), a1 = bf16_hi(aw[q]);
                const float b0 = bf16_lo(bw[q]), b1 = bf16_hi(bw[q]);
                lw[q] = pack_bf16(a0 * cs[i0] - b0 * sn[i0], a1 * cs[i1] - b1 * sn[i1]);
                hw[q] = pack_bf16(b0 * cs[i0] + a0 * sn[i0], b1 * cs[i1] + a1 * sn[i1]);
            }
        }
        *reinterpret_cast<uint4 *>(p.k_mat + dst) = lo;
        *reinterpret_cast<uint4 *>(p.k_mat + dst + kHalfDim) = hi;
    }
}

}  // namespace lazy

namespace lazy {

cudaError_t launch_kv_write(const KvWriteParams &p, cudaStream_t s) {
    kv_write_kernel<<<p.n_tok, 128, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_decode_table(const DecodeTableParams &p, cudaStream_t s) {
    const int64_t n = p.n_words * kBlockTokens;
    decode_table_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_materialize(const MaterializeParams &p, cudaStream_t s) {
    materialize_k_kernel<<<p.total_words, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace lazy
