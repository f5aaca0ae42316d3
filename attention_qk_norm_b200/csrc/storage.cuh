// storage.cuh -- 16-byte vectors of each storage type, streaming accesses,
// sub-warp sums, programmatic dependent launch and cp.async helpers.
// Part of libqknorm.so; included by qknorm.cu, the library's one translation
// unit.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace {

// ---------------------------------------------------------------- vectors --
template <typename TS>
struct Storage;

// Each storage type moves through memory in 16-byte vectors (type Vec) of
// kVec elements: 8 for bf16 / fp16, 4 for fp32, 16 for FP8.  (8-byte vectors
// for FP8, 8 elements like bf16, measured slower on B200.)
template <>
struct Storage<__nv_bfloat16> {
    using Vec = uint4;
    static constexpr int kVec = 8;  // elements per vector
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[8])
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[8])
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __nv_bfloat162 p = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
            w[i] = *reinterpret_cast<uint32_t *>(&p);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

template <>
struct Storage<float> {
    using Vec = uint4;
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[4])
    {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[4])
    {
        return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                          __float_as_uint(f[3]));
    }
};

template <>
struct Storage<__half> {
    using Vec = uint4;
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[8])
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&w[i]));
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[8])
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 p = __floats2half2_rn(f[2 * i], f[2 * i + 1]);  // round to nearest even
            w[i] = *reinterpret_cast<uint32_t *>(&p);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
    }
};

// FP8 E4M3 (bias 7, no infinities, largest finite 448): 16 per 16-byte
// vector.  Decoded exactly through fp16; encoded round-to-nearest-even,
// saturating to +-448.  The lower byte of each pair is the earlier element.
// Each 32-bit word is split into, and rebuilt from, its two 16-bit halves by
// register moves, which the conversions take and produce directly, so no
// shift or mask instruction is spent on a pair.
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float &f0, float &f1, float &f2, float &f3)
{
    asm("{\n\t.reg .b16 lo, hi, a0, a1, a2, a3;\n\t.reg .b32 h0, h1;\n\t"
        "mov.b32 {lo, hi}, %4;\n\t"
        "cvt.rn.f16x2.e4m3x2 h0, lo;\n\t"
        "cvt.rn.f16x2.e4m3x2 h1, hi;\n\t"
        "mov.b32 {a0, a1}, h0;\n\t"
        "mov.b32 {a2, a3}, h1;\n\t"
        "cvt.f32.f16 %0, a0;\n\t"
        "cvt.f32.f16 %1, a1;\n\t"
        "cvt.f32.f16 %2, a2;\n\t"
        "cvt.f32.f16 %3, a3;\n\t}"
        : "=f"(f0), "=f"(f1), "=f"(f2), "=f"(f3)
        : "r"(w));
}
__device__ __forceinline__ uint32_t f32_to_e4m3x4(float f0, float f1, float f2, float f3)
{
    uint32_t w;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"  // upper byte f1, lower byte f0
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(w)
        : "f"(f0), "f"(f1), "f"(f2), "f"(f3));
    return w;
}

template <>
struct Storage<__nv_fp8_e4m3> {
    using Vec = uint4;
    static constexpr int kVec = 16;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[16])
    {
        e4m3x4_to_f32(v.x, f[0], f[1], f[2], f[3]);
        e4m3x4_to_f32(v.y, f[4], f[5], f[6], f[7]);
        e4m3x4_to_f32(v.z, f[8], f[9], f[10], f[11]);
        e4m3x4_to_f32(v.w, f[12], f[13], f[14], f[15]);
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[16])
    {
        return make_uint4(f32_to_e4m3x4(f[0], f[1], f[2], f[3]),
                          f32_to_e4m3x4(f[4], f[5], f[6], f[7]),
                          f32_to_e4m3x4(f[8], f[9], f[10], f[11]),
                          f32_to_e4m3x4(f[12], f[13], f[14], f[15]));
    }
};

// Streaming (evict-first) vector accesses: each element is touched once.
__device__ __forceinline__ uint4 load_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void store_stream(uint4 *p, const uint4 &v) { __stcs(p, v); }

template <typename V>
__device__ __forceinline__ V zero_vec();
template <>
__device__ __forceinline__ uint4 zero_vec<uint4>() { return make_uint4(0u, 0u, 0u, 0u); }

template <int N>
__device__ __forceinline__ void load_gamma(const float *__restrict__ g, float (&out)[N])
{
    static_assert(N % 4 == 0, "gamma slices are whole float4s");
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(g) + i);
        out[4 * i] = v.x;
        out[4 * i + 1] = v.y;
        out[4 * i + 2] = v.z;
        out[4 * i + 3] = v.w;
    }
}

// Sum over an aligned group of `kWidth` lanes (a power of two dividing 32).
// With xor shuffles every lane ends with the same bits: each level adds the
// same two operands, only in swapped order, and fp32 addition commutes.
template <int kWidth>
__device__ __forceinline__ float group_sum(float s)
{
#pragma unroll
    for (int o = kWidth / 2; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    return s;
}

// Programmatic dependent launch: wait for the grids this one depends on (all
// their memory operations visible), then let dependents be scheduled.
__device__ __forceinline__ void pdl_wait_then_release()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
}

// An L2 prefetch hint for the line holding p (an address inside a buffer the
// kernel reads).  A block that starts while the grid before it is still
// draining issues these for its first rows before griddepcontrol.wait, so
// that its first loads after the wait find their lines in L2.  A prefetch
// returns no data to the thread, and every SM's accesses to a line meet in
// the L2, which the hardware keeps coherent, so a load after the wait still
// sees every write of the preceding grid.
__device__ __forceinline__ void prefetch_l2(const void *p)
{
    asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// cp.async of one 16-byte vector into shared memory (destination given as a
// shared-window address) through L2 only (.cg), in commit groups.  Each
// thread waits only for its own groups (cp.async.wait_group), which the
// hardware completes; there is no spin loop.
__device__ __forceinline__ void cp_async_s(uint32_t smem_addr, const void *gmem)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr), "l"(gmem)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---- packed fp32 pairs --
// sm_100 executes some fp32 operations on pairs of lanes held in a 64-bit
// register pair (f32x2); each lane is rounded exactly as the scalar
// instruction rounds it, so products come out bit-identical to scalar ones.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

// Sum of squares of a thread's elements.  With f32x2 the even- and the
// odd-indexed elements accumulate in the two lanes of a pair (each in
// element order), added at the end: a fixed order, the same in every kernel
// and mode that sums a head.  acc starts at f2_pack(0, 0).
template <int N>
__device__ __forceinline__ void sumsq_acc(uint64_t &acc, const float (&f)[N])
{
    static_assert(N % 2 == 0, "pairs");
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        const uint64_t x = f2_pack(f[e], f[e + 1]);
        acc = f2_fma(x, x, acc);
    }
}
__device__ __forceinline__ float sumsq_total(uint64_t acc)
{
    float a, b;
    f2_unpack(acc, a, b);
    return a + b;
}
// o[e] = a[e] * b[e] for the N elements (b through a pointer into registers
// or constants).
template <int N>
__device__ __forceinline__ void mul_elems(float (&o)[N], const float *a, const float *b)
{
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        const uint64_t p = f2_mul(f2_pack(a[e], a[e + 1]), f2_pack(b[e], b[e + 1]));
        f2_unpack(p, o[e], o[e + 1]);
    }
}
// o[e] = a[e] * c for a scalar c.
template <int N>
__device__ __forceinline__ void mul_scalar(float (&o)[N], const float *a, float c)
{
    const uint64_t cc = f2_pack(c, c);
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        const uint64_t p = f2_mul(f2_pack(a[e], a[e + 1]), cc);
        f2_unpack(p, o[e], o[e + 1]);
    }
}

// ---- mbarriers and the global timer --
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t arrivals)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(arrivals)
                 : "memory");
}
// Make initialised barriers visible to the other blocks of a cluster.
__device__ __forceinline__ void mbar_init_fence()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// One arrival plus `bytes` expected transaction bytes for the current phase.
__device__ __forceinline__ void mbar_arm(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every bounded wait gives up after this long (they complete in microseconds
// when the hardware works); each give-up is counted in g_wait_timeouts, which
// the host reads with qknorm_wait_timeouts.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ unsigned int g_wait_timeouts;

}  // namespace
