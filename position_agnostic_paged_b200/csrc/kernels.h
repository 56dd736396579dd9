// kernels.h -- parameter blocks and launch entry points shared between the
// host ABI layer (abi.cu) and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lazy_attn.h"

namespace lazy {

struct RopeTableHost {
    double theta[64];
};

constexpr int kMaxAlibiHeads = 128;   // query heads an ALiBi call may have

struct KvWriteParams {
    const uint16_t *k_raw, *v_raw;
    const int32_t *slot, *local_j;
    uint16_t *k_pool, *v_pool;
    uint32_t *blk_meta;
    int n_tok, hkv, num_blocks;
    int *d_status;
    RopeTableHost rope;
};

struct DecodeTableParams {
    const uint32_t *table;
    int64_t n_words;
    const uint32_t *blk_meta;
    int num_blocks;
    int32_t *out_block, *out_slot, *out_pos;
    int *d_status;
};

struct MaterializeParams {
    const uint32_t *table;
    const uint32_t *blk_meta;
    const uint16_t *k_pool;
    uint16_t *k_mat;
    int total_words, hkv, num_blocks;
    int *d_status;
    RopeTableHost rope;
};

struct AttnParams {
    const uint16_t *q_raw;
    const int32_t *q_pos;        // decode: [B] query position
    const int32_t *cu_q;         // prefill: [B+1]
    const int32_t *q_pos0;       // prefill: [B]
    const uint32_t *table;
    const int32_t *table_indptr;
    const uint32_t *blk_meta;
    uint16_t *out;
    float *ws_acc;               // decode: [B][Hkv][S][G][128]
    float *ws_ml;                // decode: [B][Hkv][S][G][2]
    uint16_t *q_prep;            // prefill: rotated query tiles [units][256][128] bf16, or null
    int *d_status;
    int num_req, hq, hkv, group, num_blocks, max_words;
    int words_per_split, n_splits;   // decode
    int max_q;                       // prefill
    // prefill work split: units (m-tile, KV head, request) in the order of a 3D grid
    // (m-tile fastest); units below pf_base run whole, the pf_nsplit units from pf_base run as
    // two CTAs each over the first and second half of the table's words, writing partial
    // results to ws_acc / ws_ml that prefill_combine merges
    int pf_mtiles, pf_base, pf_nsplit;
    int k_rows, v_rows;              // rows (of 128 bf16) covered by the K and V tensor maps
    float scale_log2;            // softmax scale * log2(e)
    RopeTableHost rope;          // all zero under ALiBi: every rotation is the identity
    int alibi;                   // 1: add alibi_log2[h] * (key position - query position) to each score
    float alibi_log2[kMaxAlibiHeads];   // ALiBi slope of query head h, times log2(e)
};

// Decode split plan shared by the workspace query and the launch: CTAs per (request, KV head)
// (grid_splits, each over words_per_split table words) and split partials per (request, KV
// head) (n_splits: one per CTA, or two -- one per softmax stream -- for the tensor-memory
// kernel used when a KV head serves more than 8 query heads).
struct DecodePlan {
    int words_per_split;
    int grid_splits;
    int n_splits;
};
DecodePlan decode_plan(int num_req, int hkv, int max_words, int group);
constexpr int kDecodeTcMinGroup = 9;   // query heads per KV head from which decode_tc runs

cudaError_t launch_kv_write(const KvWriteParams &p, cudaStream_t s);
cudaError_t launch_decode_table(const DecodeTableParams &p, cudaStream_t s);
cudaError_t launch_materialize(const MaterializeParams &p, cudaStream_t s);
cudaError_t launch_debug_bounded_wait(uint32_t polls, int complete, int *result, int *d_status, cudaStream_t s);
// tk8, tv8 as for the prefill (used by the tensor-memory kernel, G >= kDecodeTcMinGroup).
cudaError_t launch_decode(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                          const CUtensorMap &tv8, const AttnParams &p, bool plain, cudaStream_t s);
cudaError_t launch_decode_tc(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                             const CUtensorMap &tv8, const AttnParams &p, bool plain, cudaStream_t s);
// Merges the p.n_splits partials of every (request, query head) into the output.
cudaError_t launch_decode_combine(const AttnParams &p, cudaStream_t s);
// tk, tv: the K source and V pool as rows of 128 bf16 (one box = half of one block);
// tk8, tv8: the same memory as (d, token, head, block) (one box = half of 8 consecutive blocks);
// tq: p.q_prep as rows of 128 bf16 (one box = half of 128 rows), used when p.q_prep is set.
cudaError_t launch_prefill_tc(const CUtensorMap &tk, const CUtensorMap &tv, const CUtensorMap &tk8,
                              const CUtensorMap &tv8, const CUtensorMap &tq, const AttnParams &p, bool plain,
                              cudaStream_t s);
constexpr int kPrefillRows = 256;   // query rows per prefill CTA
// Units of the last, partial wave that are split in two when that wave is at most half full
// (one prefill CTA per SM): the grid then ends with two half-length CTAs per such unit.
inline int prefill_split_units(long long units, int sms) {
    if (units <= 0 || sms <= 0) return 0;
    const long long rem = units % sms;
    return (rem > 0 && 2 * rem <= sms) ? static_cast<int>(rem) : 0;
}
inline size_t prefill_split_bytes(int nsplit) {
    return static_cast<size_t>(nsplit) * 2 * kPrefillRows * (128 + 2) * sizeof(float);
}
// The prepared query tiles follow the split partials in the workspace, 1 KiB aligned.
inline size_t prefill_qprep_offset(int nsplit) { return (prefill_split_bytes(nsplit) + 1023) / 1024 * 1024; }
inline size_t prefill_qprep_bytes(long long units) {
    return static_cast<size_t>(units) * kPrefillRows * 128 * sizeof(uint16_t);
}

}  // namespace lazy
