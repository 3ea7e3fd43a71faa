// Device helpers shared by the qknr kernels: 128-bit streaming loads and
// stores, bf16 / E4M3 packing, warp reductions, and the fixed-point angle
// that keeps cos/sin accurate at any integer position.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace qknr {

// Read-only streaming load of 16 bytes: the input is read exactly once, so it
// bypasses L1 (the data must not be written by the same kernel).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// Streaming load that stays correct when the same kernel later overwrites the
// address (in-place use): a plain global load marked evict-first.
__device__ __forceinline__ uint4 ld_cs_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.cs.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_v2(void* p, uint2 v) {
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// bf16 pair packed in a 32-bit word: low half is the lower-addressed element.
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ void unpack8(const uint4& v, float (&f)[8]) {
    f[0] = bf16_lo(v.x); f[1] = bf16_hi(v.x);
    f[2] = bf16_lo(v.y); f[3] = bf16_hi(v.y);
    f[4] = bf16_lo(v.z); f[5] = bf16_hi(v.z);
    f[6] = bf16_lo(v.w); f[7] = bf16_hi(v.w);
}

// Round to nearest even, two floats into one bf16x2 word.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 pack8_bf16(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

// E4M3 (OCP E4M3FN), round to nearest even, saturating to +-448.
// Bytes a, b, c, d from the low end; two cvt.rn.satfinite.e4m3x2.f32 (the
// first source lands in the upper byte) joined as halves of one register.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
    uint32_t r;
    asm("{\n.reg .b16 lo, hi;\n"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n"
        "mov.b32 %0, {lo, hi};\n}"
        : "=r"(r)
        : "f"(a), "f"(b), "f"(c), "f"(d));
    return r;
}

__device__ __forceinline__ uint2 pack8_e4m3(const float (&f)[8], float scale) {
    return make_uint2(pack_e4m3x4(f[0] * scale, f[1] * scale, f[2] * scale, f[3] * scale),
                      pack_e4m3x4(f[4] * scale, f[5] * scale, f[6] * scale, f[7] * scale));
}

__device__ __forceinline__ uint2 pack8_e4m3_unscaled(const float (&f)[8]) {
    return make_uint2(pack_e4m3x4(f[0], f[1], f[2], f[3]), pack_e4m3x4(f[4], f[5], f[6], f[7]));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sum over aligned groups of G lanes (G a power of two <= 32).
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
    for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Angle of integer position `pos` for a frequency stored as a 64-bit binary
// fraction of a turn (turns_q64 = round(omega / (2 pi) * 2^64)). The product
// wraps modulo 2^64, i.e. modulo whole turns, so no precision is lost to the
// size of the angle; the top 32 bits give the signed fraction of a turn in
// [-1/2, 1/2), and sincospif turns it into cos/sin of 2 pi times that fraction.
__device__ __forceinline__ void turn_sincos(uint32_t pos, uint64_t turns_q64, float* s,
                                            float* c) {
    const uint64_t u = (uint64_t)pos * turns_q64;
    const int32_t hi = (int32_t)(u >> 32);
    const float half_turns = (float)hi * 4.656612873077392578125e-10f;  // 2^-31
    sincospif(half_turns, s, c);
}

// omega / (2 pi) as a 64-bit binary fraction of a turn, omega = base^(-2i/C).
// Positions are integers, so only the fractional part of the frequency in
// turns matters (this also covers base < 1, where omega exceeds one turn).
__device__ __forceinline__ uint64_t turns_q64(double base, int i, int C) {
    const double two_pi = 6.283185307179586476925286766559;
    const double two_64 = 18446744073709551616.0;
    double g = pow(base, -2.0 * (double)i / (double)C) / two_pi;
    g -= floor(g);
    const double x = g * two_64;
    return x >= two_64 ? 0ull : (uint64_t)x;
}

}  // namespace qknr

namespace qknr {

// ---------------------------------------------------------------------------
// Bulk asynchronous copies (TMA engine, no tensor map, no multicast) and the
// shared-memory mbarriers that track them.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

// Make initialised barriers visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Order this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy ones (a bulk copy overwriting or reading that memory).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Global -> this CTA's shared memory, completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst_smem)), "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Shared -> global bulk store, tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_u32(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until all of this thread's committed bulk stores have read their
// shared-memory source (the buffer may then be overwritten).
__device__ __forceinline__ void bulk_wait_read_all() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// Wait until all of this thread's committed bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n"
        ".reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(done)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete, giving up after `limit_ns`
// nanoseconds. Returns false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (global_timer_ns() - start > limit_ns) return false;
    }
    return true;
}

}  // namespace qknr

namespace qknr {

// Release one arrival on `bar` (plain arrive, no transaction bytes).
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Wait for phase `parity` of `bar`, giving up after `limit_ns` or as soon as
// *abort becomes non-zero. Returns false if it gave up.
__device__ __forceinline__ bool mbar_wait_abortable(uint64_t* bar, uint32_t parity,
                                                    uint64_t limit_ns,
                                                    const volatile uint32_t* abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t start = global_timer_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort != 0u) return false;
        if (global_timer_ns() - start > limit_ns) return false;
    }
    return true;
}

// Barrier over the first `nthreads` threads that arrive at named barrier `id`
// (a multiple of 32), returning whether any of them passed pred != 0.
__device__ __forceinline__ bool named_barrier_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n"
        ".reg .pred p, q;\n"
        "setp.ne.u32 q, %1, 0;\n"
        "bar.red.or.pred p, %2, %3, q;\n"
        "selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// Programmatic dependent launch. wait: block this thread until the grids this
// launch depends on have completed and their memory is visible (a no-op when
// the launch did not opt in). launch_dependents: let the next grid on the
// stream start scheduling its blocks (they still wait for this grid before
// touching memory it may write).
__device__ __forceinline__ void griddep_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Plain barrier over the first `nthreads` threads at named barrier `id`.
__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Two-lane fp32 math. On sm_100 these map to the packed fp32x2 instructions.
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(bf16_lo(w), bf16_hi(w));
}

__device__ __forceinline__ uint32_t f2_to_bf16x2(float2 v) { return pack_bf16x2(v.x, v.y); }

// The products (x_lo * w_lo, x_hi * w_hi) of two bf16 pairs, exact in fp32
// (mixed-precision FMAs with a -0 addend, which keeps the sign of a zero
// product as a plain multiply does).
__device__ __forceinline__ float2 mul_bf16x2(uint32_t x, uint32_t w) {
    float2 r;
    asm("{\n.reg .b16 xl, xh, wl, wh;\nmov.b32 {xl, xh}, %2;\nmov.b32 {wl, wh}, %3;\n"
        "fma.rn.f32.bf16 %0, xl, wl, 0f80000000;\nfma.rn.f32.bf16 %1, xh, wh, 0f80000000;\n}"
        : "=f"(r.x), "=f"(r.y)
        : "r"(x), "r"(w));
    return r;
}

// acc + (lo^2, hi^2) for the bf16 pair in w: two mixed-precision FMAs (bf16
// inputs, fp32 accumulation, one rounding each), the same results as widening
// first and one fp32x2 FMA.
__device__ __forceinline__ float2 ssq_bf16x2(uint32_t w, float2 acc) {
    asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %2;\n"
        "fma.rn.f32.bf16 %0, lo, lo, %0;\nfma.rn.f32.bf16 %1, hi, hi, %1;\n}"
        : "+f"(acc.x), "+f"(acc.y)
        : "r"(w));
    return acc;
}

// 16-bit activation pairs: bf16 (H16 = false) or IEEE binary16 (H16 = true).
template <bool H16>
__device__ __forceinline__ float2 act2_to_f2(uint32_t w) {
    if constexpr (H16) {
        return __half22float2(*reinterpret_cast<const __half2*>(&w));
    } else {
        return bf16x2_to_f2(w);
    }
}

template <bool H16>
__device__ __forceinline__ uint32_t f2_to_act2(float2 v) {
    if constexpr (H16) {
        __half2 h = __floats2half2_rn(v.x, v.y);
        return *reinterpret_cast<uint32_t*>(&h);
    } else {
        return pack_bf16x2(v.x, v.y);
    }
}

template <bool H16>
__device__ __forceinline__ float act_to_f(uint16_t b) {
    if constexpr (H16) {
        return __half2float(*reinterpret_cast<const __half*>(&b));
    } else {
        return __uint_as_float((uint32_t)b << 16);
    }
}

template <bool H16>
__device__ __forceinline__ uint16_t f_to_act(float f) {
    if constexpr (H16) {
        __half h = __float2half_rn(f);
        return *reinterpret_cast<uint16_t*>(&h);
    } else {
        __nv_bfloat16 b = __float2bfloat16_rn(f);
        return *reinterpret_cast<uint16_t*>(&b);
    }
}

}  // namespace qknr
