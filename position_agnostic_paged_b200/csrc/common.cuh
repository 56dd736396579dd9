// common.cuh -- device helpers shared by the kernels of the lazy_attn library:
// mbarriers, TMA tile loads, warp-level tensor-core fragments, bf16 packing,
// the pool's shared-memory tile layout and RoPE angle evaluation.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lazy_attn.h"

namespace lazy {

constexpr int kHeadDim = 128;
constexpr int kHalfDim = 64;
constexpr int kBlockTokens = 16;
// One 16-token block of one KV head: 16 rows x 256 B, loaded as two TMA boxes
// of 16 rows x 64 elements (128 B) with the 128-byte swizzle.
constexpr int kBoxBytes = kBlockTokens * 128;       // 2048
constexpr int kBlockBytes = 2 * kBoxBytes;          // 4096

// Bounded waits: a pipeline wait that has not completed after this many
// polls gives up, reports LAZY_DSTATUS_TIMEOUT and lets the kernel exit.
// Each poll is an mbarrier.try_wait, which itself suspends for a
// hardware-chosen time, so this bound is well above any real wait.
constexpr uint32_t kWaitPolls = 1u << 20;

// ------------------------------------------------------------------ smem addressing
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Byte offset of element (row, col) in a tile stored as two 128-byte-swizzled
// halves (cols 0-63 and 64-127) of `rows` rows each, the layout TMA writes for
// boxes of 64 bf16 x rows with CU_TENSOR_MAP_SWIZZLE_128B.  The 16-byte chunk
// index inside each 128-byte row is XOR-ed with the row index modulo 8.
__device__ __forceinline__ uint32_t swz_offset(int row, int col, int rows) {
    int half = col >> 6;
    int cb = (col & 63) * 2;
    int chunk = (cb >> 4) ^ (row & 7);
    return half * rows * 128 + row * 128 + chunk * 16 + (cb & 15);
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Non-blocking test of the phase with the given parity.
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Waits until the phase with the given parity has completed.  Returns false
// (after `polls` polls, kWaitPolls by default) if it never does.  A phase that
// has already completed is seen by one non-blocking test: measured on B200 with
// tensor memory allocated, a warp's test returns in about a third of the time
// of a potentially blocking try_wait.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint32_t polls = kWaitPolls) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < polls; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}
// Bounded wait of one role of a warp-specialised kernel that also gives up as
// soon as another role has aborted (a shared flag, checked every 256 polls).
// The role whose own wait runs out sets the flag and LAZY_DSTATUS_TIMEOUT.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                              int *d_status, uint32_t polls = kWaitPolls) {
    if (mbar_test_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < polls; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 255) == 255 && *abort_flag) return false;
    }
    *abort_flag = 1;
    if (d_status) atomicOr(d_status, LAZY_DSTATUS_TIMEOUT);
    return false;
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2D tiled load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// Loads one 16-token block (two boxes) whose first row is `row` into a 4 KiB tile.
__device__ __forceinline__ void tma_load_block(void *dst, const CUtensorMap *map, int row, uint64_t *bar) {
    tma_load_2d(dst, map, 0, row, bar);
    tma_load_2d(static_cast<uint8_t *>(dst) + kBoxBytes, map, kHalfDim, row, bar);
}

// ------------------------------------------------------------------ warp MMA (m16n8k16, bf16 -> f32)
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t x) {
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

// ------------------------------------------------------------------ numerics
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);   // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bits_to_float(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }

// Paired fp32 arithmetic (sm_100: one instruction for two lanes of work, each
// element rounded exactly as the scalar operation would round it).
// (a0, a1) += (b0, b1)
__device__ __forceinline__ void add2(float &a0, float &a1, float b0, float b1) {
    asm("{\n .reg .b64 x, y;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %3};\n add.rn.f32x2 x, x, y;\n"
        " mov.b64 {%0, %1}, x;\n}"
        : "+f"(a0), "+f"(a1)
        : "f"(b0), "f"(b1));
}
// (a0, a1) = (m * b0 + a0, m * b1 + a1)
__device__ __forceinline__ void fma2(float &a0, float &a1, float m, float b0, float b1) {
    asm("{\n .reg .b64 x, y, z;\n mov.b64 x, {%0, %1};\n mov.b64 y, {%2, %2};\n mov.b64 z, {%3, %4};\n"
        " fma.rn.f32x2 x, y, z, x;\n mov.b64 {%0, %1}, x;\n}"
        : "+f"(a0), "+f"(a1)
        : "f"(m), "f"(b0), "f"(b1));
}
// (x0, x1) = (p0 * q0 + a0, p1 * q1 + a1)
__device__ __forceinline__ void fma2v(float &x0, float &x1, float p0, float p1, float q0, float q1, float a0,
                                      float a1) {
    asm("{\n .reg .b64 p, q, a;\n mov.b64 p, {%2, %3};\n mov.b64 q, {%4, %5};\n mov.b64 a, {%6, %7};\n"
        " fma.rn.f32x2 p, p, q, a;\n mov.b64 {%0, %1}, p;\n}"
        : "=f"(x0), "=f"(x1)
        : "f"(p0), "f"(p1), "f"(q0), "f"(q1), "f"(a0), "f"(a1));
}
// (x0, x1) = (p0 * q0, p1 * q1)
__device__ __forceinline__ void mul2(float &x0, float &x1, float p0, float p1, float q0, float q1) {
    asm("{\n .reg .b64 p, q;\n mov.b64 p, {%2, %3};\n mov.b64 q, {%4, %5};\n mul.rn.f32x2 p, p, q;\n"
        " mov.b64 {%0, %1}, p;\n}"
        : "=f"(x0), "=f"(x1)
        : "f"(p0), "f"(p1), "f"(q0), "f"(q1));
}
// max(a, b, c) in one instruction (exact)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// 2^x via the SFU (PTX ex2.approx, relative error about 2^-22); 2^-inf = 0.
__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// cos and sin of delta * theta for an integer delta (|delta| < 2^31): the
// product and the reduction to [-pi, pi] are done in fp64 so that large
// relative positions keep full fp32 accuracy; the final evaluation is fp32.
__device__ __forceinline__ void rope_cos_sin(int delta, double theta, float &c, float &s) {
    const double two_pi = 6.283185307179586476925286766559;
    double a = static_cast<double>(delta) * theta;
    double k = rint(a * (1.0 / two_pi));
    float r = static_cast<float>(fma(-k, two_pi, a));
    sincosf(r, &s, &c);
}

__device__ __forceinline__ void set_status(int *d_status, int bits) {
    if (d_status) atomicOr(d_status, bits);
}

// Table word and block-metadata decoding, in registers.  The block id and the
// segment offset share one 32-bit word (gist.science, "LazyAttention: Efficient
// Retrieval-Augmented Generation with Deferred Positional Encoding", Technical
// Summary, Technical Implementation: Decoding).
__device__ __forceinline__ uint32_t word_block(uint32_t w) { return w & (LAZY_MAX_BLOCKS - 1u); }
__device__ __forceinline__ int word_offset(uint32_t w) { return static_cast<int>(w >> LAZY_BLOCK_BITS); }
__device__ __forceinline__ int meta_j0(uint32_t m) { return static_cast<int>(m >> 8) * kBlockTokens; }
__device__ __forceinline__ int meta_valid(uint32_t m) { return static_cast<int>(m & 0xFFu); }

}  // namespace lazy
