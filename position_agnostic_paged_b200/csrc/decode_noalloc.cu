// decode_noalloc.cu -- lazy_decode_attn_noalloc: the decode step for callers
// that cannot allocate device memory.
//
// lazy_decode_attn needs a caller-provided workspace for its split-K partial
// results.  Some callers have no way to provide one: a plugin that a serving
// engine hands only its input and output buffers, with no allocator to draw
// from, or code on a latency-critical path where a cudaMalloc would
// synchronise the whole device.  This entry point keeps the partials in a
// fixed array that lives in the library's own device image instead, so it
// allocates nothing.  The caller still passes every input and output.
//
// The array costs every GPU that loads the library kStaticScratchBytes of
// device memory until the process exits, and it is shared by all calls, so
// calls that may run at the same time on the GPU (other streams, other host
// threads) race on it and must be serialised by the caller.
#include <cuda_runtime.h>

#include <mutex>

#include "lazy_attn.h"

namespace {

// 16 MiB: enough for the split-K partials of 128 requests x 8 KV heads x 8
// query heads per KV head at two splits (the decode shapes of Llama-3.1-70B),
// or 64 requests with 4 splits at the 8B shapes.
constexpr size_t kStaticScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

// Device-side scratch.  In host code this name is only a stand-in for the
// symbol: its device address comes from cudaGetSymbolAddress below.
__device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

std::mutex g_mu;
struct ScratchAddr {
    void *ctx = nullptr;    // the context the address was looked up in
    void *addr = nullptr;
};
ScratchAddr g_scratch_addr[kMaxDevices];

typedef int (*CtxGetCurrentFn)(void **);

// The driver's cuCtxGetCurrent, found once through the runtime (no link-time
// dependency on libcuda); null if the driver does not provide it.
CtxGetCurrentFn ctx_get_current() {
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(ptr);
    });
    return fn;
}

// Device address of the scratch array in the current device's current
// context.  It is looked up once per context (the first call on a device does
// this set-up) and looked up again when the context changes -- after a
// cudaDeviceReset the module may load at another address.  Without the
// driver's context query the address is looked up on every call.
int scratch_for_current_device(void **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LAZY_ECUDA;
    void *ctx = nullptr;
    CtxGetCurrentFn get = ctx_get_current();
    const bool have_ctx = get && get(&ctx) == 0 && ctx;
    std::lock_guard<std::mutex> lock(g_mu);
    ScratchAddr &e = g_scratch_addr[dev];
    if (!have_ctx || !e.addr || e.ctx != ctx) {
        void *ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return LAZY_ECUDA;
        e.addr = ptr;
        e.ctx = have_ctx ? ctx : nullptr;
    }
    *out = e.addr;
    return LAZY_OK;
}

}  // namespace

extern "C" size_t lazy_decode_noalloc_capacity(void) { return kStaticScratchBytes; }

extern "C" int lazy_decode_attn_noalloc(const lazy_attn_cfg *cfg, const uint16_t *q_raw, const int32_t *q_pos,
                                        int num_req, const uint32_t *table, const int32_t *table_indptr,
                                        int max_words, const uint32_t *blk_meta, const uint16_t *k_pool,
                                        const uint16_t *v_pool, int num_blocks, uint16_t *out, int *d_status,
                                        void *stream) {
    // size check first, on the host: nothing is launched for a request that does not fit
    if (cfg && num_req > 0 && max_words > 0) {
        const size_t need = lazy_decode_workspace_bytes(cfg, num_req, max_words);
        if (need > kStaticScratchBytes) return LAZY_ERANGE;
    }
    void *scratch = nullptr;
    const int rc = scratch_for_current_device(&scratch);
    if (rc != LAZY_OK) return rc;
    // Every split of every (request, KV head) writes its partial (an empty
    // split writes m = -inf, l = 0 and a zero accumulator) before the combine
    // reads it, so the leftover contents of an earlier call need no clearing.
    return lazy_decode_attn(cfg, q_raw, q_pos, num_req, table, table_indptr, max_words, blk_meta, k_pool, v_pool,
                            num_blocks, out, scratch, kStaticScratchBytes, d_status, stream);
}
