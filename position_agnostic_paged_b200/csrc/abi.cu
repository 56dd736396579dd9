// abi.cu -- the extern "C" entry points declared in include/lazy_attn.h:
// argument validation on the host, the RoPE frequency table, TMA tensor maps
// over the caller's pools, and kernel launches.  No device memory is
// allocated here; every buffer belongs to the caller.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "kernels.h"
#include "lazy_attn.h"

using namespace lazy;

namespace {

constexpr int kVersion = 102;

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// A pool (or materialised copy) viewed as rows of 128 bf16 (256 B); boxes of
// box_rows rows x 64 elements with the 128-byte swizzle (by default one half of a
// 16-token block).
bool make_rows_map(CUtensorMap *map, const void *base, int64_t rows, int box_rows = 16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows <= 0) return false;
    cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {256};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same pool viewed as (d, token, head, block): one box covers `box_blocks`
// consecutive blocks of one head and one 64-element half (2 KiB per block), laid
// out in shared memory exactly like that many single-block boxes stacked.
bool make_blocks_map(CUtensorMap *map, const void *base, int64_t nblocks, int hkv, int box_blocks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || nblocks <= 0 || hkv <= 0) return false;
    cuuint64_t dims[4] = {128, 16, static_cast<cuuint64_t>(hkv), static_cast<cuuint64_t>(nblocks)};
    cuuint64_t strides[3] = {256, 4096, static_cast<cuuint64_t>(hkv) * 4096};
    cuuint32_t box[4] = {64, 16, 1, static_cast<cuuint32_t>(box_blocks)};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Streaming multiprocessors of the current device (0 if it cannot be queried).
int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

int check_cfg(const lazy_attn_cfg *cfg) {
    if (!cfg) return LAZY_EINVAL;
    if (cfg->head_dim != 128 || cfg->block_size != 16) return LAZY_ESHAPE;
    if (cfg->num_kv_heads <= 0 || cfg->num_q_heads <= 0) return LAZY_ESHAPE;
    if (cfg->num_q_heads % cfg->num_kv_heads != 0) return LAZY_ESHAPE;
    if (cfg->num_q_heads / cfg->num_kv_heads > 32) return LAZY_ESHAPE;
    if (cfg->num_kv_heads > 64) return LAZY_ESHAPE;
    if (!(cfg->rope_base > 1.0f) || !std::isfinite(cfg->rope_base)) return LAZY_EINVAL;
    if (cfg->rope_theta)
        for (int i = 0; i < 64; ++i)
            if (!std::isfinite(cfg->rope_theta[i]) || cfg->rope_theta[i] < 0.0) return LAZY_EINVAL;
    if (cfg->alibi_slopes) {
        if (cfg->num_q_heads > kMaxAlibiHeads) return LAZY_ESHAPE;
        for (int h = 0; h < cfg->num_q_heads; ++h)
            if (!std::isfinite(cfg->alibi_slopes[h])) return LAZY_EINVAL;
    }
    return LAZY_OK;
}

void fill_rope(RopeTableHost &t, const lazy_attn_cfg *cfg) {
    // theta_i for the rotate-half pairs (i, i + d/2): the caller's table, else base^(-2i/d);
    // under ALiBi all zero, so that every rotation (pool write, query) is exactly the identity
    for (int i = 0; i < 64; ++i)
        t.theta[i] = cfg->alibi_slopes ? 0.0
                     : cfg->rope_theta ? cfg->rope_theta[i]
                                       : std::pow(static_cast<double>(cfg->rope_base), -2.0 * i / 128.0);
}

float scale_log2(const lazy_attn_cfg *cfg) {
    const double s = cfg->softmax_scale > 0.f ? cfg->softmax_scale : 1.0 / std::sqrt(128.0);
    return static_cast<float>(s * 1.4426950408889634);   // log2(e)
}

int launch_rc(cudaError_t e) { return e == cudaSuccess ? LAZY_OK : LAZY_ECUDA; }

size_t decode_ws(const lazy_attn_cfg *cfg, int num_req, int max_words) {
    const DecodePlan pl = decode_plan(num_req, cfg->num_kv_heads, max_words, cfg->num_q_heads / cfg->num_kv_heads);
    const size_t parts = static_cast<size_t>(num_req) * cfg->num_kv_heads * pl.n_splits *
                         (cfg->num_q_heads / cfg->num_kv_heads);
    return parts * (128 + 2) * sizeof(float);
}

int attn_common(const lazy_attn_cfg *cfg, AttnParams &p, int num_req, const uint32_t *table,
                const int32_t *table_indptr, int max_words, const uint32_t *blk_meta, const uint16_t *v_pool,
                int num_blocks, uint16_t *out, int *d_status) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (num_req < 0 || max_words < 0 || num_blocks < 0) return LAZY_EINVAL;
    if (num_req > 0 && (!table_indptr || !out || !blk_meta || !v_pool)) return LAZY_EINVAL;
    if (max_words > 0 && !table) return LAZY_EINVAL;
    if (static_cast<uint32_t>(num_blocks) > LAZY_MAX_BLOCKS) return LAZY_ERANGE;
    std::memset(&p, 0, sizeof p);
    p.table = table;
    p.table_indptr = table_indptr;
    p.blk_meta = blk_meta;
    p.out = out;
    p.d_status = d_status;
    p.num_req = num_req;
    p.hq = cfg->num_q_heads;
    p.hkv = cfg->num_kv_heads;
    p.group = cfg->num_q_heads / cfg->num_kv_heads;
    p.num_blocks = num_blocks;
    p.max_words = max_words;
    p.scale_log2 = scale_log2(cfg);
    fill_rope(p.rope, cfg);
    p.alibi = cfg->alibi_slopes ? 1 : 0;
    for (int h = 0; h < cfg->num_q_heads && cfg->alibi_slopes; ++h)
        p.alibi_log2[h] = static_cast<float>(cfg->alibi_slopes[h] * 1.4426950408889634);   // log2(e)
    return LAZY_OK;
}

int decode_impl(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos, int num_req,
                const uint32_t *table, const int32_t *table_indptr, int max_words, const uint32_t *blk_meta,
                const uint16_t *k_src, int64_t k_rows, const uint16_t *v_pool, int num_blocks, uint16_t *out,
                void *workspace, size_t ws_bytes, int *d_status, void *stream, bool plain, bool dry = false) {
    AttnParams p;
    int rc = attn_common(cfg, p, num_req, table, table_indptr, max_words, blk_meta, v_pool, num_blocks, out,
                         d_status);
    if (rc) return rc;
    if (num_req == 0) return LAZY_OK;
    if (!q_raw || !q_pos || !k_src) return LAZY_EINVAL;
    if (max_words == 0 || num_blocks == 0 || k_rows == 0) {
        if (dry) return LAZY_OK;
        // nothing can be visible: every output row is zero
        return launch_rc(cudaMemsetAsync(out, 0, static_cast<size_t>(num_req) * p.hq * 128 * 2,
                                         static_cast<cudaStream_t>(stream)));
    }
    const size_t need = decode_ws(cfg, num_req, max_words);
    if (!workspace || ws_bytes < need) return LAZY_EWORKSPACE;
    if (dry) return LAZY_OK;
    const DecodePlan pl = decode_plan(num_req, cfg->num_kv_heads, max_words, p.group);
    p.q_raw = q_raw;
    p.q_pos = q_pos;
    p.k_rows = static_cast<int>(k_rows);
    p.v_rows = static_cast<int>(static_cast<int64_t>(num_blocks) * p.hkv * 16);
    p.words_per_split = pl.words_per_split;
    p.n_splits = pl.n_splits;
    const size_t parts = static_cast<size_t>(num_req) * p.hkv * pl.n_splits * p.group;
    p.ws_acc = static_cast<float *>(workspace);
    p.ws_ml = p.ws_acc + parts * 128;
    CUtensorMap tk, tv, tk8, tv8;
    if (!make_rows_map(&tk, k_src, k_rows) || !make_rows_map(&tv, v_pool, p.v_rows)) return LAZY_ECUDA;
    if (!make_blocks_map(&tk8, k_src, k_rows / (16 * p.hkv), p.hkv, 8) ||
        !make_blocks_map(&tv8, v_pool, num_blocks, p.hkv, 8))
        return LAZY_ECUDA;
    return launch_rc(launch_decode(tk, tv, tk8, tv8, p, plain, static_cast<cudaStream_t>(stream)));
}

int prefill_impl(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *cu_q, const int32_t *q_pos0,
                 int num_req, int total_q, int max_q, const uint32_t *table, const int32_t *table_indptr,
                 int max_words, const uint32_t *blk_meta, const uint16_t *k_src, int64_t k_rows,
                 const uint16_t *v_pool, int num_blocks, uint16_t *out, void *workspace, size_t ws_bytes,
                 int *d_status, void *stream, bool plain, bool dry = false) {
    AttnParams p;
    int rc = attn_common(cfg, p, num_req, table, table_indptr, max_words, blk_meta, v_pool, num_blocks, out,
                         d_status);
    if (rc) return rc;
    if (total_q < 0 || max_q < 0) return LAZY_EINVAL;
    if (num_req == 0 || total_q == 0 || max_q == 0) return LAZY_OK;
    if (!q_raw || !cu_q || !q_pos0 || !k_src) return LAZY_EINVAL;
    if (static_cast<int64_t>(max_q) * p.group > (int64_t(1) << 30)) return LAZY_ERANGE;
    if (max_words == 0 || num_blocks == 0 || k_rows == 0) {
        if (dry) return LAZY_OK;
        return launch_rc(cudaMemsetAsync(out, 0, static_cast<size_t>(total_q) * p.hq * 128 * 2,
                                         static_cast<cudaStream_t>(stream)));
    }
    p.q_raw = q_raw;
    p.cu_q = cu_q;
    p.q_pos0 = q_pos0;
    p.max_q = max_q;
    // work units and, with a large enough workspace, the split of the last partial wave
    p.pf_mtiles = static_cast<int>((static_cast<int64_t>(max_q) * p.group + kPrefillRows - 1) / kPrefillRows);
    const long long units = static_cast<long long>(p.pf_mtiles) * p.hkv * num_req;
    if (units > (1LL << 30)) return LAZY_ERANGE;
    if (dry) return LAZY_OK;
    int nsplit = prefill_split_units(units, sm_count());
    if (!workspace || ws_bytes < prefill_split_bytes(nsplit)) nsplit = 0;
    p.pf_nsplit = nsplit;
    p.pf_base = static_cast<int>(units) - nsplit;
    p.ws_acc = static_cast<float *>(workspace);
    p.ws_ml = nsplit ? p.ws_acc + static_cast<size_t>(nsplit) * 2 * kPrefillRows * 128 : nullptr;
    // with room after the split partials (16-byte aligned, as TMA requires), the query tiles
    // are rotated by a first kernel and loaded by TMA; otherwise each CTA rotates its own
    const size_t qoff = prefill_qprep_offset(nsplit);
    if (workspace && ws_bytes >= qoff + prefill_qprep_bytes(units) && units * kPrefillRows <= INT32_MAX &&
        (reinterpret_cast<uintptr_t>(workspace) + qoff) % 16 == 0)
        p.q_prep = reinterpret_cast<uint16_t *>(static_cast<char *>(workspace) + qoff);
    p.k_rows = static_cast<int>(k_rows);
    p.v_rows = static_cast<int>(static_cast<int64_t>(num_blocks) * p.hkv * 16);
    CUtensorMap tk, tv, tk8, tv8, tq;
    if (!make_rows_map(&tk, k_src, k_rows) || !make_rows_map(&tv, v_pool, p.v_rows)) return LAZY_ECUDA;
    if (!make_blocks_map(&tk8, k_src, k_rows / (16 * p.hkv), p.hkv, 8) ||
        !make_blocks_map(&tv8, v_pool, num_blocks, p.hkv, 8))
        return LAZY_ECUDA;
    if (p.q_prep) {
        if (!make_rows_map(&tq, p.q_prep, units * kPrefillRows, 128)) return LAZY_ECUDA;
    } else {
        tq = tk;   // not read
    }
    // each request writes exactly its own query tokens' rows
    return launch_rc(launch_prefill_tc(tk, tv, tk8, tv8, tq, p, plain, static_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

int lazy_version(void) { return kVersion; }

const char *lazy_strerror(int code) {
    switch (code) {
    case LAZY_OK: return "ok";
    case LAZY_EINVAL: return "invalid argument (null pointer or negative count)";
    case LAZY_ERANGE: return "value out of range (table field, pool size or count too large)";
    case LAZY_ESHAPE: return "unsupported shape (head_dim must be 128, block_size 16, Hq/Hkv an integer <= 32)";
    case LAZY_EWORKSPACE: return "workspace too small";
    case LAZY_ECUDA: return "CUDA launch or driver call failed";
    default: return "unknown error";
    }
}

int lazy_pack_words(const int32_t *block, const int32_t *offset, int64_t n, uint32_t *words) {
    if (n < 0) return LAZY_EINVAL;
    if (n > 0 && (!block || !offset || !words)) return LAZY_EINVAL;
    for (int64_t i = 0; i < n; ++i) {
        if (block[i] < 0 || static_cast<uint32_t>(block[i]) >= LAZY_MAX_BLOCKS) return LAZY_ERANGE;
        if (offset[i] < 0 || static_cast<uint32_t>(offset[i]) > LAZY_MAX_OFFSET) return LAZY_ERANGE;
        words[i] = lazy_pack(static_cast<uint32_t>(block[i]), static_cast<uint32_t>(offset[i]));
    }
    return LAZY_OK;
}

int lazy_kv_write(const lazy_attn_cfg *cfg, const uint16_t *k_raw, const uint16_t *v_raw, int n_tok,
                  const int32_t *slot, const int32_t *local_j, uint16_t *k_pool, uint16_t *v_pool,
                  uint32_t *blk_meta, int num_blocks, int *d_status, void *stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (n_tok < 0 || num_blocks < 0) return LAZY_EINVAL;
    if (static_cast<uint32_t>(num_blocks) > LAZY_MAX_BLOCKS) return LAZY_ERANGE;
    if (n_tok == 0) return LAZY_OK;
    if (!k_raw || !v_raw || !slot || !local_j || !k_pool || !v_pool || !blk_meta) return LAZY_EINVAL;
    KvWriteParams p;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.slot = slot;
    p.local_j = local_j;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.blk_meta = blk_meta;
    p.n_tok = n_tok;
    p.hkv = cfg->num_kv_heads;
    p.num_blocks = num_blocks;
    p.d_status = d_status;
    fill_rope(p.rope, cfg);
    return launch_rc(launch_kv_write(p, static_cast<cudaStream_t>(stream)));
}

size_t lazy_decode_workspace_bytes(const lazy_attn_cfg *cfg, int num_req, int max_words) {
    if (check_cfg(cfg) != LAZY_OK || num_req <= 0 || max_words <= 0) return 0;
    return decode_ws(cfg, num_req, max_words);
}

int lazy_decode_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos, int num_req,
                     const uint32_t *table, const int32_t *table_indptr, int max_words, const uint32_t *blk_meta,
                     const uint16_t *k_pool, const uint16_t *v_pool, int num_blocks, uint16_t *out, void *workspace,
                     size_t ws_bytes, int *d_status, void *stream) {
    if (cfg && check_cfg(cfg) == LAZY_OK && num_req > 0 && num_blocks > 0 && !k_pool) return LAZY_EINVAL;
    const int64_t rows = cfg ? static_cast<int64_t>(num_blocks) * (cfg->num_kv_heads > 0 ? cfg->num_kv_heads : 0) * 16 : 0;
    return decode_impl(cfg, q_raw, q_pos, num_req, table, table_indptr, max_words, blk_meta, k_pool, rows, v_pool,
                       num_blocks, out, workspace, ws_bytes, d_status, stream, false);
}

size_t lazy_prefill_workspace_bytes(const lazy_attn_cfg *cfg, int num_req, int total_q, int max_q, int max_words) {
    (void)total_q;
    (void)max_words;
    if (!cfg || check_cfg(cfg) != LAZY_OK || num_req <= 0 || max_q <= 0) return 0;
    const int G = cfg->num_q_heads / cfg->num_kv_heads;
    const long long mtiles = (static_cast<long long>(max_q) * G + kPrefillRows - 1) / kPrefillRows;
    const long long units = mtiles * cfg->num_kv_heads * num_req;
    return prefill_qprep_offset(prefill_split_units(units, sm_count())) + prefill_qprep_bytes(units);
}

int lazy_prefill_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *cu_q, const int32_t *q_pos0,
                      int num_req, int total_q, int max_q, const uint32_t *table, const int32_t *table_indptr,
                      int max_words, const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool,
                      int num_blocks, uint16_t *out, void *workspace, size_t ws_bytes, int *d_status, void *stream) {
    if (cfg && check_cfg(cfg) == LAZY_OK && num_req > 0 && num_blocks > 0 && !k_pool) return LAZY_EINVAL;
    const int64_t rows = cfg ? static_cast<int64_t>(num_blocks) * (cfg->num_kv_heads > 0 ? cfg->num_kv_heads : 0) * 16 : 0;
    return prefill_impl(cfg, q_raw, cu_q, q_pos0, num_req, total_q, max_q, table, table_indptr, max_words, blk_meta,
                        k_pool, rows, v_pool, num_blocks, out, workspace, ws_bytes, d_status, stream, false);
}

int lazy_mixed_attn(const lazy_attn_cfg *cfg, const lazy_prefill_batch *pf, const lazy_decode_batch *dc,
                    const uint32_t *blk_meta, const uint16_t *k_pool, const uint16_t *v_pool, int num_blocks,
                    int *d_status, void *stream) {
    const bool has_pf = pf && pf->num_req > 0, has_dc = dc && dc->num_req > 0;
    if (has_pf && has_dc && pf->workspace && dc->workspace && pf->workspace == dc->workspace) return LAZY_EINVAL;
    if (cfg && check_cfg(cfg) == LAZY_OK && (has_pf || has_dc) && num_blocks > 0 && !k_pool) return LAZY_EINVAL;
    const int64_t rows = cfg ? static_cast<int64_t>(num_blocks) * (cfg->num_kv_heads > 0 ? cfg->num_kv_heads : 0) * 16 : 0;
    // both batches are checked before anything is enqueued
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (has_pf) {
        rc = prefill_impl(cfg, pf->q_raw, pf->cu_q, pf->q_pos0, pf->num_req, pf->total_q, pf->max_q, pf->table,
                          pf->table_indptr, pf->max_words, blk_meta, k_pool, rows, v_pool, num_blocks, pf->out,
                          pf->workspace, pf->ws_bytes, d_status, stream, false, true);
        if (rc) return rc;
    }
    if (has_dc) {
        rc = decode_impl(cfg, dc->q_raw, dc->q_pos, dc->num_req, dc->table, dc->table_indptr, dc->max_words,
                         blk_meta, k_pool, rows, v_pool, num_blocks, dc->out, dc->workspace, dc->ws_bytes, d_status,
                         stream, false, true);
        if (rc) return rc;
    }
    // Both run in order on the caller's stream.  Running them concurrently (the prefill on a
    // second stream of higher priority, the decode on the SMs its grid leaves idle) measured 3-5 %
    // slower than this order, with small and large prefill batches alike.
    if (has_pf) {
        rc = prefill_impl(cfg, pf->q_raw, pf->cu_q, pf->q_pos0, pf->num_req, pf->total_q, pf->max_q, pf->table,
                          pf->table_indptr, pf->max_words, blk_meta, k_pool, rows, v_pool, num_blocks, pf->out,
                          pf->workspace, pf->ws_bytes, d_status, stream, false);
        if (rc) return rc;
    }
    if (has_dc)
        return decode_impl(cfg, dc->q_raw, dc->q_pos, dc->num_req, dc->table, dc->table_indptr, dc->max_words,
                           blk_meta, k_pool, rows, v_pool, num_blocks, dc->out, dc->workspace, dc->ws_bytes,
                           d_status, stream, false);
    return LAZY_OK;
}

int lazy_materialize_k(const lazy_attn_cfg *cfg, const uint32_t *table, int total_words, const uint32_t *blk_meta,
                       const uint16_t *k_pool, int num_blocks, uint16_t *k_mat, int *d_status, void *stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->alibi_slopes) return LAZY_EINVAL;   // ALiBi keys carry no position to materialise
    if (total_words < 0 || num_blocks < 0) return LAZY_EINVAL;
    if (static_cast<uint32_t>(num_blocks) > LAZY_MAX_BLOCKS) return LAZY_ERANGE;
    if (total_words == 0) return LAZY_OK;
    if (!table || !blk_meta || !k_pool || !k_mat) return LAZY_EINVAL;
    MaterializeParams p;
    p.table = table;
    p.blk_meta = blk_meta;
    p.k_pool = k_pool;
    p.k_mat = k_mat;
    p.total_words = total_words;
    p.hkv = cfg->num_kv_heads;
    p.num_blocks = num_blocks;
    p.d_status = d_status;
    fill_rope(p.rope, cfg);
    return launch_rc(launch_materialize(p, static_cast<cudaStream_t>(stream)));
}

int lazy_plain_decode_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos, int num_req,
                           const uint32_t *table, const int32_t *table_indptr, int max_words,
                           const uint32_t *blk_meta, const uint16_t *k_mat, int total_words, const uint16_t *v_pool,
                           int num_blocks, uint16_t *out, void *workspace, size_t ws_bytes, int *d_status,
                           void *stream) {
    if (total_words < 0 || (cfg && cfg->alibi_slopes)) return LAZY_EINVAL;
    if (cfg && check_cfg(cfg) == LAZY_OK && num_req > 0 && total_words > 0 && !k_mat) return LAZY_EINVAL;
    const int64_t rows = cfg ? static_cast<int64_t>(total_words) * (cfg->num_kv_heads > 0 ? cfg->num_kv_heads : 0) * 16 : 0;
    if (rows >= (int64_t(1) << 31)) return LAZY_ERANGE;
    return decode_impl(cfg, q_raw, q_pos, num_req, table, table_indptr, max_words, blk_meta, k_mat, rows, v_pool,
                       num_blocks, out, workspace, ws_bytes, d_status, stream, true);
}

int lazy_plain_prefill_attn(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *cu_q,
                            const int32_t *q_pos0, int num_req, int total_q, int max_q, const uint32_t *table,
                            const int32_t *table_indptr, int max_words, const uint32_t *blk_meta,
                            const uint16_t *k_mat, int total_words, const uint16_t *v_pool, int num_blocks,
                            uint16_t *out, void *workspace, size_t ws_bytes, int *d_status, void *stream) {
    if (total_words < 0 || (cfg && cfg->alibi_slopes)) return LAZY_EINVAL;
    if (cfg && check_cfg(cfg) == LAZY_OK && num_req > 0 && total_words > 0 && !k_mat) return LAZY_EINVAL;
    const int64_t rows = cfg ? static_cast<int64_t>(total_words) * (cfg->num_kv_heads > 0 ? cfg->num_kv_heads : 0) * 16 : 0;
    if (rows >= (int64_t(1) << 31)) return LAZY_ERANGE;
    return prefill_impl(cfg, q_raw, cu_q, q_pos0, num_req, total_q, max_q, table, table_indptr, max_words, blk_meta,
                        k_mat, rows, v_pool, num_blocks, out, workspace, ws_bytes, d_status, stream, true);
}

int lazy_debug_decode_table(const uint32_t *table, int64_t n_words, const uint32_t *blk_meta, int num_blocks,
                            int32_t *out_block, int32_t *out_slot, int32_t *out_pos, int *d_status, void *stream) {
    if (n_words < 0 || num_blocks < 0) return LAZY_EINVAL;
    if (n_words == 0) return LAZY_OK;
    if (!table || !blk_meta || !out_block || !out_slot || !out_pos) return LAZY_EINVAL;
    if (n_words > (int64_t(1) << 26)) return LAZY_ERANGE;
    DecodeTableParams p;
    p.table = table;
    p.n_words = n_words;
    p.blk_meta = blk_meta;
    p.num_blocks = num_blocks;
    p.out_block = out_block;
    p.out_slot = out_slot;
    p.out_pos = out_pos;
    p.d_status = d_status;
    return launch_rc(launch_decode_table(p, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
