// qknorm.cu -- QK-Norm kernels for B200 (sm_100a) and the C ABI of
// libqknorm.so (declared in include/qknorm.h).
//
// Both operations are HBM-bound streams: every Q/K element is read once and
// written once, with ~3 flops per element, far below the ridge point, so no
// tensor cores are involved.  The design goals are full 16-byte vector
// accesses, enough bytes in flight per SM to cover HBM latency, and a grid
// sized to the resident capacity of the 148 SMs.
//
// Per-head (sglang PR #13189, Motivation / Modifications; RMSNorm definition
// from the SwiftQK review, core_discovery): one sub-warp of LPR lanes owns a
// (token, head) row of D elements.  Each lane holds D/kVec/LPR vectors of
// the row, sums squares in fp32, and the sub-warp reduces with
// xor shuffles.  Every thread keeps two rows in flight per iteration and its
// slice of gamma_q / gamma_k in registers for the whole launch.
//
// Layerwise (SwiftQK abstract; review key_machinery): a persistent block
// walks tokens with a grid stride.  Each thread copies its vectors of
// the next token into a two-stage shared-memory ring with cp.async while it
// works on the current one.  The per-head partial sums of squares meet in
// shared memory behind one barrier; then each warp, for the vectors (q, k)
// its threads hold, forms every emulated shard's fp32 partial from that
// shard's heads alone and combines the shard scalars, and every thread scales
// its vectors, re-read from the ring, by the inverse RMS of its vector.
//
// Both kernels are launched with programmatic dependent launch: they wait on
// griddepcontrol.wait before their first global memory access, so a kernel
// earlier in the stream always finishes first, and they allow the next
// kernel to be scheduled as soon as all of their blocks are resident.  No
// kernel here waits on another block, so none can hang.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "qknorm.h"

namespace {

constexpr int kMaxDevices = 64;

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
template <>
struct Storage<__nv_fp8_e4m3> {
    using Vec = uint4;
    static constexpr int kVec = 16;
    __device__ __forceinline__ static void unpack(const uint4 &v, float (&f)[16])
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(
                    (__nv_fp8x2_storage_t)((w[i] >> (16 * j)) & 0xffffu), __NV_E4M3);
                const float2 p = __half22float2(*reinterpret_cast<const __half2 *>(&r));
                f[4 * i + 2 * j] = p.x;
                f[4 * i + 2 * j + 1] = p.y;
            }
        }
    }
    __device__ __forceinline__ static uint4 pack(const float (&f)[16])
    {
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i], f[4 * i + 1]),
                                                         __NV_SATFINITE, __NV_E4M3);
            const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(f[4 * i + 2], f[4 * i + 3]),
                                                         __NV_SATFINITE, __NV_E4M3);
            w[i] = lo | (hi << 16);
        }
        return make_uint4(w[0], w[1], w[2], w[3]);
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

// cp.async of one 16-byte vector into shared memory through L2 only (.cg),
// in commit groups.  Each thread waits only for its own groups
// (cp.async.wait_group), which the hardware completes; there is no spin loop.
template <int kBytes>
__device__ __forceinline__ void cp_async(void *smem, const void *gmem)
{
    static_assert(kBytes == 16, "vectors are 16 bytes");
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ---------------------------------------------------------------- per-head --
constexpr int kPerHeadThreads = 256;
constexpr int kPerHeadRowsInFlight = 2;
// Resident 256-thread blocks per SM that the register budget must allow, by
// elements a lane holds per row: six (40 registers) for the single-weight
// loop with 8 elements, five (48) with both weights; four (64) and three (80)
// for FP8's 16 elements; four for fp32 D=256 (two vectors per lane).  Each
// fits without spilling.
template <typename TS, int D, bool kHasK>
constexpr int per_head_min_blocks()
{
    constexpr int kNV = D / Storage<TS>::kVec;
    constexpr int kVPL = kNV > 32 ? kNV / 32 : 1;
    constexpr int kEPL = kVPL * Storage<TS>::kVec;
    return kVPL > 1 ? 4 : (kEPL > 8 ? (kHasK ? 3 : 4) : (kHasK ? 5 : 6));
}

// Rows are visited with a grid stride: thread group g takes rows g, g + G,
// g + 2G, ... (G groups in the grid), U at a time.  The (token, head) pair of
// each of its U rows is found once by division and then advanced by the fixed
// step U*G with an add and one wrap, so the loop does no integer division.
//
// kSplit (used for FP8 with both kinds of heads): blocks [0, q_blocks) walk
// the query rows only and the other blocks the key rows only, each with one
// weight slice; holding both slices and selecting per element needs 80
// registers for FP8's 16 elements per lane, one block per SM fewer.
template <typename TS, int D, int U, bool kHasK, bool kSplit = false>
__global__ void __launch_bounds__(kPerHeadThreads, (per_head_min_blocks<TS, D, kHasK>()))
qkn_per_head_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, uint32_t heads,
                    uint32_t Hq, const float *__restrict__ gamma_q,
                    const float *__restrict__ gamma_k, float eps, uint32_t q_blocks)
{
    static_assert(!(kSplit && kHasK), "a split block holds one weight");
    using S = Storage<TS>;
    using V = typename S::Vec;
    constexpr int kVec = S::kVec;
    constexpr int kNV = D / kVec;                  // vectors per row
    constexpr int kLPR = kNV < 32 ? kNV : 32;      // lanes per row
    constexpr int kVPL = kNV / kLPR;               // vectors per lane per row
    constexpr int kEPL = kVPL * kVec;              // elements per lane per row
    static_assert(32 % kLPR == 0 && kNV % kLPR == 0, "row must map onto a sub-warp");

    pdl_wait_then_release();
    uint64_t block = blockIdx.x, nblocks = gridDim.x;
    if constexpr (kSplit) {
        if (blockIdx.x >= q_blocks) {  // key rows: the columns after the Hq query heads
            qkv += (int64_t)Hq * D;
            gamma_q = gamma_k;
            heads -= Hq;
            block -= q_blocks;
            nblocks -= q_blocks;
        } else {
            heads = Hq;
            nblocks = q_blocks;
        }
    }
    const uint64_t tid = block * blockDim.x + threadIdx.x;
    const uint32_t lane = (uint32_t)(tid % kLPR);
    const uint64_t group = tid / kLPR;
    const uint64_t ngroups = (nblocks * blockDim.x) / kLPR;

    // This lane's columns are fixed: vectors lane, lane + LPR, ... of a row.
    float gq[kEPL], gk[kHasK ? kEPL : 1];
#pragma unroll
    for (int v = 0; v < kVPL; ++v) {
        const int col = (lane + v * kLPR) * kVec;
        float tq[kVec];
        load_gamma<kVec>(gamma_q + col, tq);
#pragma unroll
        for (int e = 0; e < kVec; ++e) gq[v * kVec + e] = tq[e];
        if constexpr (kHasK) {
            float tk[kVec];
            load_gamma<kVec>(gamma_k + col, tk);
#pragma unroll
            for (int e = 0; e < kVec; ++e) gk[v * kVec + e] = tk[e];
        }
    }

    // The first rows and the step are below U * ngroups (at most a few
    // hundred thousand), so 32-bit division can find their (token, head)
    // pairs; it shortens the start of the single-weight kernel (measured
    // 1.4% at the 48-head, 4096-token shape), while the two-weight variant
    // measured faster with 64-bit division.
    int64_t t[U];
    uint32_t h[U];
    const uint64_t step = ngroups * U;
    int64_t dt;
    uint32_t dh;
    if constexpr (!kHasK) {
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const uint32_t r = (uint32_t)(k * ngroups + group);
            const uint32_t q = r / heads;
            t[k] = q;
            h[k] = r - q * heads;
        }
        const uint32_t dt32 = (uint32_t)step / heads;
        dt = dt32;
        dh = (uint32_t)step - dt32 * heads;
    } else {
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const uint64_t r = (uint64_t)k * ngroups + group;
            t[k] = (int64_t)(r / heads);
            h[k] = (uint32_t)(r - (uint64_t)t[k] * heads);
        }
        dt = (int64_t)(step / heads);
        dh = (uint32_t)(step - (uint64_t)dt * heads);
    }
    const uint64_t rows = (uint64_t)T * heads;
    // The trip count is the same for every thread, so whole warps reach each
    // shuffle together; rows past the end contribute zeros and store nothing.
    for (uint64_t base = 0; base < rows; base += step) {
        V x[U][kVPL];
        V *ptr[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            ptr[k] = reinterpret_cast<V *>(qkv + t[k] * row_stride + (int64_t)h[k] * D) + lane;
#pragma unroll
            for (int v = 0; v < kVPL; ++v)
                x[k][v] = t[k] < T ? load_stream(ptr[k] + v * kLPR) : zero_vec<V>();
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
            float f[kVPL][kVec];
            float s = 0.f;
#pragma unroll
            for (int v = 0; v < kVPL; ++v) {
                S::unpack(x[k][v], f[v]);
#pragma unroll
                for (int e = 0; e < kVec; ++e) s = fmaf(f[v][e], f[v][e], s);
            }
            s = group_sum<kLPR>(s);
            const float rinv = rsqrtf(s / (float)D + eps);
            if (t[k] < T) {
                const bool is_q = !kHasK || h[k] < Hq;
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    float o[kVec];
#pragma unroll
                    for (int e = 0; e < kVec; ++e) {
                        float g = gq[v * kVec + e];
                        if constexpr (kHasK) g = is_q ? g : gk[v * kVec + e];
                        o[e] = f[v][e] * rinv * g;
                    }
                    store_stream(ptr[k] + v * kLPR, S::pack(o));
                }
            }
            h[k] += dh;
            t[k] += dt;
            if (h[k] >= heads) {
                h[k] -= heads;
                t[k] += 1;
            }
        }
    }
}

// --------------------------------------------------------------- layerwise --
constexpr int kLayerwiseStages = 2;

// How warp_sumsq reduces the nh head partials of one vector (q or k).  The
// host fills it once per launch, so the token loop divides nothing.
//   used:      lanes that hold partials, min(p, 32) with p the largest power
//              of two dividing nh (0 when nh == 0);
//   per_lane:  heads each of those lanes sums, in order (nh / used);
//   per_shard: lanes per emulated shard (used / nshards).
struct SumPlan {
    int used;
    int per_lane;
    int per_shard;
};

// Sum of squares of one vector from its head partials part[0..nh), computed
// by one whole warp; every lane returns the same value.
//
// The reduction tree is fixed by nh alone: lane i sums heads
// [i*per_lane, (i+1)*per_lane) in order, then xor butterflies join lanes at
// distance 1, 2, 4, ...  With n shards (n a power of two dividing nh, so
// n <= used), shard r holds exactly lanes [r*used/n, (r+1)*used/n): the
// butterflies below distance used/n form each shard's partial S_r from that
// shard's heads only, and the remaining ones are the scalar combine of
// S_0..S_{n-1}.  So the result does not depend on n, bit for bit.
__device__ __forceinline__ float warp_sumsq(const float *part, const SumPlan &p, int lane)
{
    float v = 0.f;
    if (lane < p.used)
        for (int j = 0; j < p.per_lane; ++j) v += part[lane * p.per_lane + j];
    for (int o = 1; o < p.per_shard; o <<= 1)  // rank-local partial S_r
        v += __shfl_xor_sync(0xffffffffu, v, o);
    for (int o = p.per_shard; o < p.used; o <<= 1)  // combine of the shard scalars
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return __shfl_sync(0xffffffffu, v, 0);
}

// ---- cluster exchange of head partials (transaction barriers) --
// Each block of a cluster keeps two mbarriers, one per partials buffer.  The
// owner of a head pushes that head's fp32 partial into the buffer of every
// block of the cluster with st.async, which also counts its 4 bytes against
// the receiving block's barrier; a block's barrier phase completes once all
// (Hq + Hk) partials of the token have landed and its own thread 0 has armed
// the phase.  No cluster-wide barrier and no memory fence is on the token path.
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t arrivals)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(arrivals)
                 : "memory");
}
// Make the initialised barriers visible to the other blocks of the cluster.
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
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// The shared::cluster address of `cta_addr` (a shared::cta address) in the
// block of cluster rank `rank`.
__device__ __forceinline__ uint32_t cluster_addr(uint32_t cta_addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(cta_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_async_f32(uint32_t dst, float v, uint32_t bar)
{
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(
                     dst),
                 "r"(__float_as_uint(v)), "r"(bar)
                 : "memory");
}
__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits on a barrier give up after this long (they complete in microseconds
// when the exchange works); each give-up is counted in g_wait_timeouts.
constexpr uint64_t kWaitLimitNs = 2000000000ull;
__device__ unsigned int g_wait_timeouts;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > kWaitLimitNs) return false;
    return true;
}

// What a layerwise launch does with a token.
//   kFused:    partial sums, scalar combine, inverse RMS and scaling, in place.
//   kPartials: only this rank's two fp32 sums of squares (its q heads, its k
//              heads), written to aux[2t], aux[2t+1]; the data is not written.
//   kApply:    only the scaling, by 1/sqrt(aux[2t]/len_q + eps) for q and
//              1/sqrt(aux[2t+1]/len_k + eps) for k, where aux holds the sums
//              over all ranks and len_q, len_k the full vector lengths.
// The mean S/L is formed as S * inv_len with inv_len = 1/L rounded to fp32
// once per launch.
enum LayerwiseMode { kFused = 0, kPartials = 1, kApply = 2 };

// A token's heads are split over the CL blocks of a thread-block cluster
// (CL = 1 for a plain launch): block c of a cluster owns heads
// [c*hc, (c+1)*hc), hc = heads/CL, with roundup32(hc * NV / VPT) threads;
// thread (h, l) owns vectors l, l + LPH, ... of head h (LPH = NV / VPT lanes
// per head), and thread l == 0 is the head's owner.  Dynamic shared memory
// per block: kLayerwiseStages stages of this block's part of a token
// (hc*D*sizeof(TS) bytes), two buffers of `heads` fp32 head partials
// (alternating per token), then the two exchange barriers (CL > 1).  With
// CL = 1 the partials meet behind one block barrier per token; with CL > 1
// each owner pushes its partial into every block of the cluster and each
// block waits on its own barrier (see the exchange helpers above).
template <typename TS, int D, int VPT, bool kGammaRegs, bool kCluster, int kMode, bool kOverlap>
__device__ __forceinline__ void
layerwise_tokens(TS *__restrict__ qkv, int64_t row_stride, int64_t T, int Hq, int Hk,
                 const float *__restrict__ gamma_q, const float *__restrict__ gamma_k, float eps,
                 float inv_len_q, float inv_len_k, SumPlan plan_q, SumPlan plan_k,
                 float *__restrict__ aux)
{
    using S = Storage<TS>;
    using V = typename S::Vec;
    constexpr int kVB = (int)sizeof(V);  // bytes per vector
    constexpr int kVec = S::kVec;
    constexpr int kNV = D / kVec;     // vectors per head
    constexpr int kLPH = kNV / VPT;   // threads per head
    constexpr int kEPT = VPT * kVec;  // elements per thread
    constexpr int NST = kLayerwiseStages;
    constexpr bool kExchange = kCluster && kMode != kApply;
    // Vector loops unroll fully when gamma sits in registers (indexed by v);
    // with gamma in L1 the long loops unroll by 8.
    constexpr int kUnroll = kGammaRegs || VPT < 8 ? VPT : 8;
    static_assert(kNV % VPT == 0 && 32 % kLPH == 0, "head must map onto a sub-warp");

    extern __shared__ __align__(16) unsigned char smem[];
    const int heads = Hq + Hk;
    int cl = 1, crank = 0;
    if constexpr (kCluster) {
        cl = (int)cooperative_groups::this_cluster().num_blocks();
        crank = (int)cooperative_groups::this_cluster().block_rank();
    }
    const int hc = heads / cl;           // heads of this block
    const int h_lo = crank * hc;
    const int span = hc * D * (int)sizeof(TS);
    float *part = reinterpret_cast<float *>(smem + (size_t)NST * span);
    uint64_t *bar = reinterpret_cast<uint64_t *>(part + 2 * heads);
    const uint32_t token_bytes = (uint32_t)heads * (uint32_t)sizeof(float);
    const int hl = threadIdx.x / kLPH;   // head within this block
    const int h = h_lo + hl;
    const int l = threadIdx.x % kLPH;
    const bool active = hl < hc;
    const int lane = threadIdx.x % 32;
    // Heads of this warp's threads; a warp computes only the inverse RMS of
    // the vectors it holds (warp-uniform, so whole warps shuffle together).
    const int warp_first_head = h_lo + (threadIdx.x & ~31) / kLPH;
    const int warp_last_head = h_lo + (threadIdx.x | 31) / kLPH;
    const bool need_q = warp_first_head < Hq;
    const bool need_k = Hk > 0 && warp_last_head >= Hq;
    const int64_t first = blockIdx.x / cl, stride = gridDim.x / cl;  // this cluster's tokens

    pdl_wait_then_release();
    // This thread's head weights (the partials step has none).
    const float *gb = gamma_q;
    if (kMode != kPartials && active)
        gb = h < Hq ? gamma_q + (int64_t)h * D : gamma_k + (int64_t)(h - Hq) * D;
    float g[kGammaRegs ? kEPT : 1];
#pragma unroll
    for (int e = 0; e < (kGammaRegs ? kEPT : 1); ++e) g[e] = 0.f;
    if (kGammaRegs && kMode != kPartials && active) {
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            float t4[kVec];
            load_gamma<kVec>(gb + (l + v * kLPH) * kVec, t4);
#pragma unroll
            for (int e = 0; e < kVec; ++e) g[v * kVec + e] = t4[e];
        }
    }
    const int64_t col0 = (int64_t)h * D;          // in the token row
    const int scol0 = (hl * D + l * kVec) * (int)sizeof(TS);  // in a stage
    // Each thread copies, and later reads, only its own vectors of a stage.
    auto fetch = [&](int64_t tok, int st) {
        if (active && tok < T) {
            const V *src = reinterpret_cast<const V *>(qkv + tok * row_stride + col0);
            V *dst = reinterpret_cast<V *>(smem + (size_t)st * span + scol0);
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v) cp_async<kVB>(dst + v * kLPH, src + l + v * kLPH);
        }
        cp_async_commit();
    };
#pragma unroll
    for (int i = 0; i < NST - 1; ++i) fetch(first + (int64_t)i * stride, i);
    if constexpr (kExchange) {
        if (threadIdx.x == 0) {
            mbar_init(&bar[0], 1);
            mbar_init(&bar[1], 1);
            mbar_init_fence();
            mbar_arm(&bar[0], token_bytes);
            mbar_arm(&bar[1], token_bytes);
        }
        // Distributed shared memory may only be touched once every block of
        // the cluster is running: meet once, barriers initialised and armed,
        // before the first remote write.
        cooperative_groups::this_cluster().sync();
    }
    int st = 0;
    uint32_t it = 0;  // tokens this block has done; partials buffer it % 2
    bool timed_out = false;
    for (int64_t t = first; t < T; t += stride, ++it) {
        // Refill the stage this thread finished with on the previous token.
        fetch(t + (int64_t)(NST - 1) * stride, (st + NST - 1) % NST);
        cp_async_wait<NST - 1>();
        const V *sp = reinterpret_cast<const V *>(smem + (size_t)st * span + scol0);
        float rq = 0.f, rk = 0.f;
        float xg[kOverlap ? kEPT : 1];  // x * gamma, formed before the combine
        if constexpr (kMode == kApply) {
            // Sums over all ranks come in; no exchange inside the launch.
            if (Hq > 0) rq = rsqrtf(__ldg(aux + 2 * t) * inv_len_q + eps);
            if (Hk > 0) rk = rsqrtf(__ldg(aux + 2 * t + 1) * inv_len_k + eps);
        } else {
            float s = 0.f;
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v) {
                float f[kVec];
                S::unpack(active ? sp[v * kLPH] : zero_vec<V>(), f);
#pragma unroll
                for (int e = 0; e < kVec; ++e) s = fmaf(f[e], f[e], s);
                if constexpr (kOverlap) {
#pragma unroll
                    for (int e = 0; e < kVec; ++e) xg[v * kVec + e] = f[e] * g[v * kVec + e];
                }
            }
            s = group_sum<kLPH>(s);
            // Partials alternate between two buffers.  The next write into
            // this token's buffer is for the token after next; every block
            // sends it only after the token in between, which needs a partial
            // from every warp of the cluster, and each warp sends that only
            // after it has finished reading this buffer.  (Every warp holds an
            // owner: its first thread.)
            const uint32_t pb = it & 1u;
            float *pp = part + pb * heads;
            if constexpr (kExchange) {
                if (active && l == 0) {
                    const uint32_t dst = smem_u32(pp + h), b = smem_u32(&bar[pb]);
                    for (int r = 0; r < cl; ++r)
                        st_async_f32(cluster_addr(dst, (uint32_t)r), s,
                                     cluster_addr(b, (uint32_t)r));
                }
                // Buffer pb serves every other token: phase it/2 of its barrier.
                if (!timed_out && !mbar_wait_bounded(&bar[pb], (it >> 1) & 1u)) {
                    timed_out = true;
                    if (lane == 0) atomicAdd(&g_wait_timeouts, 1u);
                }
                // Arm the barrier's next phase (the token after next) before this
                // thread sends its next partial, which any sender of that phase
                // has to wait for.
                if (threadIdx.x == 0 && !timed_out) mbar_arm(&bar[pb], token_bytes);
            } else {
                if (active && l == 0) pp[h] = s;
                __syncthreads();
            }
            if constexpr (kMode == kPartials) {
                // One warp of the cluster's first block writes this rank's sums.
                if (threadIdx.x < 32 && crank == 0) {
                    const float sq = warp_sumsq(pp, plan_q, lane);
                    const float sk = warp_sumsq(pp + Hq, plan_k, lane);
                    if (lane == 0) {
                        aux[2 * t] = sq;
                        aux[2 * t + 1] = sk;
                    }
                }
            } else {
                if (need_q) rq = rsqrtf(warp_sumsq(pp, plan_q, lane) * inv_len_q + eps);
                if (need_k) rk = rsqrtf(warp_sumsq(pp + Hq, plan_k, lane) * inv_len_k + eps);
            }
        }
        if (kMode != kPartials && active) {
            const float rinv = h < Hq ? rq : rk;
            V *p = reinterpret_cast<V *>(qkv + t * row_stride + col0);
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v) {
                float o[kVec];
                if constexpr (kOverlap) {
#pragma unroll
                    for (int e = 0; e < kVec; ++e) o[e] = xg[v * kVec + e] * rinv;
                } else {
                    float f[kVec], gv[kVec];
                    S::unpack(sp[v * kLPH], f);
                    if constexpr (kGammaRegs) {
#pragma unroll
                        for (int e = 0; e < kVec; ++e) gv[e] = g[v * kVec + e];
                    } else {
                        load_gamma<kVec>(gb + (l + v * kLPH) * kVec, gv);
                    }
#pragma unroll
                    for (int e = 0; e < kVec; ++e) o[e] = f[e] * gv[e] * rinv;
                }
                store_stream(p + l + v * kLPH, S::pack(o));
            }
        }
        st = (st + 1 == NST) ? 0 : st + 1;
    }
    cp_async_wait<0>();
    // No block leaves while a partner could still write into it.
    if constexpr (kExchange) cooperative_groups::this_cluster().sync();
}

// Registers per thread: 40, 48 or 56 when a thread keeps 8, 16 or 32
// elements (and as many gamma values) per token.  The caps fit without
// spilling and leave room for more resident blocks than the compiler's own
// choice (up to 64); measured on B200 they are the fastest for every storage
// type and head_dim.  The overlap variant also keeps the thread's x * gamma
// products across the combine: 48, 64 or 96.
#ifndef QKN_LW_REGS8
#define QKN_LW_REGS8 40
#endif
#ifndef QKN_LW_REGS16
#define QKN_LW_REGS16 48
#endif
#ifndef QKN_LW_REGS32
#define QKN_LW_REGS32 56
#endif
#ifndef QKN_LW_OVERLAP_REGS8
#define QKN_LW_OVERLAP_REGS8 48
#endif
#ifndef QKN_LW_OVERLAP_REGS16
#define QKN_LW_OVERLAP_REGS16 64
#endif
#ifndef QKN_LW_OVERLAP_REGS32
#define QKN_LW_OVERLAP_REGS32 96
#endif
__host__ __device__ constexpr int layerwise_regs(int ept, bool overlap)
{
    return overlap ? (ept <= 8 ? QKN_LW_OVERLAP_REGS8
                               : (ept <= 16 ? QKN_LW_OVERLAP_REGS16 : QKN_LW_OVERLAP_REGS32))
                   : (ept <= 8 ? QKN_LW_REGS8 : (ept <= 16 ? QKN_LW_REGS16 : QKN_LW_REGS32));
}

// Gamma in registers (at most 32 elements per thread).  kOverlap: each
// thread forms x * gamma while the token's partials are still being
// combined (SwiftQK's overlap of the weight multiplication with the
// exchange), so after the combine only the multiplication by the inverse RMS
// remains, without a second pass over the staged token.
template <typename TS, int D, int VPT, bool kCluster, int kMode, bool kOverlap>
__global__ void __maxnreg__((layerwise_regs(VPT * Storage<TS>::kVec, kOverlap)))
qkn_layerwise_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, int Hq, int Hk,
                     const float *__restrict__ gamma_q, const float *__restrict__ gamma_k,
                     float eps, float inv_len_q, float inv_len_k, SumPlan plan_q,
                     SumPlan plan_k, float *__restrict__ aux)
{
    layerwise_tokens<TS, D, VPT, true, kCluster, kMode, kOverlap>(
        qkv, row_stride, T, Hq, Hk, gamma_q, gamma_k, eps, inv_len_q, inv_len_k, plan_q, plan_k,
        aux);
}

// Gamma read through L1 (tokens too wide for registers; one block per token,
// up to 1024 threads).
template <typename TS, int D, int VPT, int kMode>
__global__ void __launch_bounds__(1024)
qkn_layerwise_l1_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, int Hq, int Hk,
                        const float *__restrict__ gamma_q, const float *__restrict__ gamma_k,
                        float eps, float inv_len_q, float inv_len_k, SumPlan plan_q,
                        SumPlan plan_k, float *__restrict__ aux)
{
    layerwise_tokens<TS, D, VPT, false, false, kMode, false>(qkv, row_stride, T, Hq, Hk, gamma_q,
                                                             gamma_k, eps, inv_len_q, inv_len_k,
                                                             plan_q, plan_k, aux);
}

// ------------------------------------------------------------------- host --
thread_local int g_last_cuda_error = 0;

int cuda_fail(cudaError_t e)
{
    g_last_cuda_error = (int)e;
    return QKN_ERR_CUDA;
}

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;  // max dynamic shared memory per block (opt-in)
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

int device_info(int *dev_out, DeviceInfo *info)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return QKN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev[dev].sms == 0) {
        int n = 0, smem = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        g_dev[dev].sms = n;
        g_dev[dev].smem_optin = smem;
    }
    *dev_out = dev;
    *info = g_dev[dev];
    return QKN_OK;
}

// Launch with programmatic stream serialization allowed (see the kernels'
// griddepcontrol.wait) and, when cluster > 1, as clusters of `cluster`
// blocks along x; then report the launch status.
template <typename... Params, typename... Args>
int launch_pdl(void (*kern)(Params...), unsigned grid, unsigned threads, size_t smem,
               cudaStream_t stream, unsigned cluster, Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = cluster > 1 ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, args...);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int elem_size(int dtype)
{
    switch (dtype) {
    case QKN_BF16: return 2;
    case QKN_FP32: return 4;
    case QKN_FP16: return 2;
    case QKN_FP8_E4M3: return 1;
    default: return 0;
    }
}

// Checks shared by both entry points.  Order: dtype, shape, eps, T == 0,
// pointers, alignment.
int validate(const void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
             const float *gamma_q, const float *gamma_k, float eps, bool *nothing_to_do)
{
    *nothing_to_do = false;
    const int es = elem_size(dtype);
    if (es == 0) return QKN_ERR_UNSUPPORTED;
    if (T < 0 || Hq < 0 || Hk < 0 || Hq + Hk < 1 || row_stride < 0) return QKN_ERR_SHAPE;
    if (D != 64 && D != 128 && D != 256) return QKN_ERR_UNSUPPORTED;
    const int64_t W = ((int64_t)Hq + 2 * (int64_t)Hk) * D;
    if (row_stride < W) return QKN_ERR_SHAPE;
    if (!(eps >= 0.f) || !isfinite(eps)) return QKN_ERR_EPS;
    if (T == 0) {
        *nothing_to_do = true;
        return QKN_OK;
    }
    if (T > INT64_MAX / (row_stride > 0 ? row_stride : 1) / es) return QKN_ERR_SHAPE;
    if (qkv == nullptr) return QKN_ERR_NULL;
    if (Hq > 0 && gamma_q == nullptr) return QKN_ERR_NULL;
    if (Hk > 0 && gamma_k == nullptr) return QKN_ERR_NULL;
    if (!aligned16(qkv) || ((row_stride * es) & 15) != 0) return QKN_ERR_ALIGN;
    if ((gamma_q != nullptr && !aligned16(gamma_q)) || (gamma_k != nullptr && !aligned16(gamma_k)))
        return QKN_ERR_ALIGN;
    return QKN_OK;
}

// Per-kernel, per-device set-up done once: the opt-in dynamic shared-memory
// limit, and (for kernels without dynamic shared memory) the resident blocks
// per SM at the block size in use.
struct KernelCache {
    std::atomic<int> per_sm[kMaxDevices][33] = {};
    std::atomic<uint64_t> smem_ready{0};
};

template <typename Kern>
int resident_blocks(Kern kern, KernelCache &kc, int dev, const DeviceInfo &info, int threads,
                    size_t smem, int *out)
{
    if (smem > 48 * 1024 && !(kc.smem_ready.load(std::memory_order_acquire) & (1ull << dev))) {
        const cudaError_t e = cudaFuncSetAttribute(
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, info.smem_optin);
        if (e != cudaSuccess) return cuda_fail(e);
        kc.smem_ready.fetch_or(1ull << dev, std::memory_order_acq_rel);
    }
    const int slot = threads / 32;
    int n = smem == 0 ? kc.per_sm[dev][slot].load(std::memory_order_relaxed) : 0;
    if (n == 0) {
        const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
        if (e != cudaSuccess) return cuda_fail(e);
        if (smem == 0) kc.per_sm[dev][slot].store(n, std::memory_order_relaxed);
    }
    *out = n;
    return QKN_OK;
}

template <typename TS, int D, bool kHasK, bool kSplit = false>
int launch_per_head_k(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride, const float *gq,
                      const float *gk, float eps, cudaStream_t stream)
{
    constexpr int U = kPerHeadRowsInFlight;
    constexpr int kNV = D / Storage<TS>::kVec;
    constexpr int kLPR = kNV < 32 ? kNV : 32;
    auto kern = qkn_per_head_kernel<TS, D, U, kHasK, kSplit>;
    static KernelCache kc;
    int dev = 0, per_sm = 0, rc;
    DeviceInfo info;
    if ((rc = device_info(&dev, &info)) != QKN_OK) return rc;
    if ((rc = resident_blocks(kern, kc, dev, info, kPerHeadThreads, 0, &per_sm)) != QKN_OK)
        return rc;
    if (per_sm < 1) return QKN_ERR_UNSUPPORTED;
    const uint64_t rows_per_block = (uint64_t)(kPerHeadThreads / kLPR) * U;
    uint64_t cap = (uint64_t)info.sms * per_sm;
    const uint64_t rows = (uint64_t)T * (uint64_t)(Hq + Hk);
    uint64_t grid = (rows + rows_per_block - 1) / rows_per_block, q_blocks = 0;
    if constexpr (kSplit) {
        // Blocks per segment: as many as its rows need; when both together
        // exceed the resident capacity, the capacity split in proportion to
        // the rows, at least one block each.
        const uint64_t rq = (uint64_t)T * (uint64_t)Hq, rk = (uint64_t)T * (uint64_t)Hk;
        uint64_t bq = (rq + rows_per_block - 1) / rows_per_block;
        uint64_t bk = (rk + rows_per_block - 1) / rows_per_block;
        if (cap < 2) cap = 2;
        if (bq + bk > cap) {
            bq = (cap * rq + (rq + rk) / 2) / (rq + rk);
            if (bq < 1) bq = 1;
            if (bq > cap - 1) bq = cap - 1;
            bk = cap - bq;
        }
        grid = bq + bk;
        q_blocks = bq;
    } else if (grid > cap) {
        grid = cap;
    }
    return launch_pdl(kern, (unsigned)grid, kPerHeadThreads, 0, stream, 1u,
                      static_cast<TS *>(qkv), row_stride, T, (uint32_t)(Hq + Hk), (uint32_t)Hq, gq,
                      gk, eps, (uint32_t)q_blocks);
}

template <typename TS, int D>
int launch_per_head(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride, const float *gq,
                    const float *gk, float eps, cudaStream_t stream)
{
    if (Hq > 0 && Hk > 0) {
        if constexpr (Storage<TS>::kVec == 16)  // FP8
            return launch_per_head_k<TS, D, false, true>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,
                                                          stream);
        else
            return launch_per_head_k<TS, D, true>(qkv, T, Hq, Hk, row_stride, gq, gk, eps, stream);
    }
    const float *g = Hq > 0 ? gq : gk;
    return launch_per_head_k<TS, D, false>(qkv, T, Hq, Hk, row_stride, g, nullptr, eps, stream);
}

// A layerwise kernel variant exists when a head splits into whole vectors
// per thread on at most 32 lanes.  Gamma stays in registers up to 32
// elements per thread, else it is read through L1 when scaling.
template <typename TS, int D, int VPT>
constexpr bool layerwise_vpt_ok()
{
    constexpr int kNV = D / Storage<TS>::kVec;
    return kNV % VPT == 0 && kNV / VPT <= 32;
}

template <typename TS, int VPT>
constexpr bool layerwise_gamma_regs()
{
    return VPT * Storage<TS>::kVec <= 32;
}

template <typename TS, int D, int VPT, bool kCluster, int kMode, bool kOverlap = false>
int launch_layerwise_vpt(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride,
                         const float *gq, const float *gk, float eps, int threads, int cluster,
                         float inv_len_q, float inv_len_k, SumPlan plan_q, SumPlan plan_k,
                         float *aux, cudaStream_t stream)
{
    auto kern = [] {
        if constexpr (layerwise_gamma_regs<TS, VPT>())
            return qkn_layerwise_kernel<TS, D, VPT, kCluster, kMode, kOverlap>;
        else
            return qkn_layerwise_l1_kernel<TS, D, VPT, kMode>;
    }();
    static KernelCache kc;
    const int heads = Hq + Hk;
    const size_t span = (size_t)(heads / cluster) * D * sizeof(TS);
    const size_t smem =
        kLayerwiseStages * span + (size_t)2 * heads * sizeof(float) + 2 * sizeof(uint64_t);
    int dev = 0, rc;
    DeviceInfo info;
    if ((rc = device_info(&dev, &info)) != QKN_OK) return rc;
    if (smem > (size_t)info.smem_optin) return QKN_ERR_UNSUPPORTED;
    int64_t cap = 0;  // co-resident clusters (of `cluster` blocks) on the device
    if (kCluster) {
        if (smem > 48 * 1024 && !(kc.smem_ready.load(std::memory_order_acquire) & (1ull << dev))) {
            const cudaError_t e = cudaFuncSetAttribute(
                kern, cudaFuncAttributeMaxDynamicSharedMemorySize, info.smem_optin);
            if (e != cudaSuccess) return cuda_fail(e);
            kc.smem_ready.fetch_or(1ull << dev, std::memory_order_acq_rel);
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)cluster);
        cfg.blockDim = dim3((unsigned)threads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)cluster;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        const cudaError_t e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess) return cuda_fail(e);
        cap = n;
    } else {
        int per_sm = 0;
        if ((rc = resident_blocks(kern, kc, dev, info, threads, smem, &per_sm)) != QKN_OK) return rc;
        cap = (int64_t)info.sms * per_sm;
    }
    if (cap < 1) return QKN_ERR_UNSUPPORTED;
    const int64_t clusters = T < cap ? T : cap;
    return launch_pdl(kern, (unsigned)(clusters * cluster), threads, smem, stream,
                      (unsigned)cluster, static_cast<TS *>(qkv), row_stride, T, Hq, Hk, gq, gk,
                      eps, inv_len_q, inv_len_k, plan_q, plan_k, aux);
}

// Launch shape, chosen from measurements on B200 over the four storage types,
// head_dim 64 to 256 and 40 to 72 heads:
//  * the smallest cluster size CL (1, 2, 4 or 8 blocks, dividing the head
//    count) for which some vectors-per-thread count VPT keeps gamma in
//    registers (VPT * kVec <= 32) and the block within 576 threads;
//  * the fewest such VPT, but at least 2: with one vector per thread the
//    per-token work of a thread is too short for its fixed per-token cost;
//  * on short inputs, fewer than 12 tokens per resident cluster, twice that
//    VPT when gamma still fits: half the threads per block, about twice the
//    resident blocks, so more tokens are under way at once.
// If no cluster size fits, one block per token with the fewest VPT within
// 1024 threads, gamma read through L1 where it does not fit registers.
// For fp32 and FP8 storage, a fused launch that keeps its VPT and is not
// short by the overlap variant's own (larger) register count runs that
// variant: it saves the second pass over the staged token, whose cost per
// element is highest there (4 elements per 16-byte read for fp32, 16
// conversions for FP8).  Measured on B200 it gained 1-13% on those shapes;
// for bf16 and fp16 and on short inputs its extra registers cost more than
// the pass.
constexpr int kLayerwiseMaxThreads = 576;
constexpr int kLayerwiseShortTokens = 12;
constexpr int kMaxCluster = 8;

template <typename TS>
constexpr bool layerwise_overlap_type()
{
    return Storage<TS>::kVec == 4 || Storage<TS>::kVec == 16;  // fp32, FP8
}

// Resident blocks per SM by the register file and the thread limit; the
// shape rule's estimate (the launch itself queries the occupancy).
int layerwise_blocks_estimate(int threads, int regs)
{
    const int by_regs = 65536 / (threads * ((regs + 7) / 8 * 8));
    const int by_threads = 2048 / threads;
    const int n = by_regs < by_threads ? by_regs : by_threads;
    return n < 32 ? n : 32;
}

// The reduction plan of warp_sumsq for nh head partials split into nshards.
SumPlan sum_plan(int nh, int nshards)
{
    SumPlan p = {0, 0, 0};
    if (nh > 0) {
        const int p2 = nh & (-nh);
        p.used = p2 < 32 ? p2 : 32;
        p.per_lane = nh / p.used;
        p.per_shard = p.used / nshards;  // nshards is a power of two dividing nh
    }
    return p;
}

// len_q, len_k: the normalised lengths (the full vectors; for kFused and
// kPartials they are this launch's own Hq*D and Hk*D).
template <typename TS, int D, int kMode = kFused>
int launch_layerwise(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride, const float *gq,
                     const float *gk, float eps, int nshards, cudaStream_t stream,
                     float len_q = -1.f, float len_k = -1.f, float *aux = nullptr)
{
    if (len_q < 0.f) len_q = (float)((int64_t)Hq * D);  // exact: spans are < 2^24 elements
    if (len_k < 0.f) len_k = (float)((int64_t)Hk * D);
    const float inv_len_q = Hq > 0 ? 1.0f / len_q : 0.f;
    const float inv_len_k = Hk > 0 ? 1.0f / len_k : 0.f;
    const SumPlan plan_q = sum_plan(Hq, nshards), plan_k = sum_plan(Hk, nshards);
    constexpr int kNV = D / Storage<TS>::kVec;
    constexpr int kVec = Storage<TS>::kVec;
    const int64_t heads = Hq + Hk;
    auto vpt_ok = [](int vpt) { return vpt <= kNV && kNV % vpt == 0 && kNV / vpt <= 32; };
    auto threads_for = [&](int cl, int vpt) {
        return (int)(((heads / cl * (kNV / vpt)) + 31) / 32 * 32);
    };
    int chosen = 0, cluster = 1;
    for (int cl = 1; cl <= kMaxCluster && chosen == 0; cl *= 2) {
        if (heads % cl != 0) continue;
        for (int vpt = 2; vpt * kVec <= 32; vpt *= 2) {
            if (vpt_ok(vpt) && threads_for(cl, vpt) <= kLayerwiseMaxThreads) {
                chosen = vpt;
                cluster = cl;
                break;
            }
        }
    }
    bool overlap = false;
    if (chosen != 0) {
        int dev = 0, rc;
        DeviceInfo info;
        if ((rc = device_info(&dev, &info)) != QKN_OK) return rc;
        // Resident clusters (token pipelines) with `regs` registers per thread.
        auto pipelines = [&](int regs) {
            const int per_sm = layerwise_blocks_estimate(threads_for(cluster, chosen), regs);
            return (int64_t)info.sms * per_sm / cluster;
        };
        const int ept = chosen * kVec;
        const bool can_double = 2 * ept <= 32 && vpt_ok(2 * chosen);
        if (can_double && T < kLayerwiseShortTokens * pipelines(layerwise_regs(ept, false)))
            chosen *= 2;
        else if (kMode == kFused && layerwise_overlap_type<TS>())
            overlap = T >= kLayerwiseShortTokens * pipelines(layerwise_regs(ept, true));
    }
    for (int vpt = 1; vpt <= kNV && chosen == 0; vpt *= 2)
        if (vpt_ok(vpt) && threads_for(1, vpt) <= 1024) chosen = vpt;
    if (chosen == 0) return QKN_ERR_UNSUPPORTED;
    const int threads = (int)(((heads / cluster * (kNV / chosen)) + 31) / 32 * 32);
    constexpr bool kMayOverlap = kMode == kFused && layerwise_overlap_type<TS>();
#define QKN_LW_CASE(V)                                                                         \
    case V:                                                                                    \
        if constexpr (layerwise_vpt_ok<TS, D, V>()) {                                          \
            if constexpr (layerwise_gamma_regs<TS, V>()) {                                     \
                if constexpr (kMayOverlap) {                                                   \
                    if (overlap && cluster > 1)                                                \
                        return launch_layerwise_vpt<TS, D, V, true, kMode, true>(              \
                            qkv, T, Hq, Hk, row_stride, gq, gk, eps, threads, cluster,         \
                            inv_len_q, inv_len_k, plan_q, plan_k, aux, stream);                \
                    if (overlap)                                                               \
                        return launch_layerwise_vpt<TS, D, V, false, kMode, true>(             \
                            qkv, T, Hq, Hk, row_stride, gq, gk, eps, threads, 1, inv_len_q,    \
                            inv_len_k, plan_q, plan_k, aux, stream);                           \
                }                                                                              \
                if (cluster > 1)                                                               \
                    return launch_layerwise_vpt<TS, D, V, true, kMode>(                        \
                        qkv, T, Hq, Hk, row_stride, gq, gk, eps, threads, cluster, inv_len_q,  \
                        inv_len_k, plan_q, plan_k, aux, stream);                               \
            }                                                                                  \
            return launch_layerwise_vpt<TS, D, V, false, kMode>(                               \
                qkv, T, Hq, Hk, row_stride, gq, gk, eps, threads, 1, inv_len_q, inv_len_k,     \
                plan_q, plan_k, aux, stream);                                                  \
        }                                                                                      \
        break;
    switch (chosen) {
        QKN_LW_CASE(1)
        QKN_LW_CASE(2)
        QKN_LW_CASE(4)
        QKN_LW_CASE(8)
        QKN_LW_CASE(16)
        QKN_LW_CASE(32)
        QKN_LW_CASE(64)
    default:
        break;
    }
#undef QKN_LW_CASE
    return QKN_ERR_UNSUPPORTED;
}

// Storage type and head_dim as template arguments of F::run.
template <typename F, typename... Args>
int dispatch(int dtype, int D, Args... args)
{
#define QKN_BY_D(TS)                                                                           \
    switch (D) {                                                                               \
    case 64: return F::template run<TS, 64>(args...);                                          \
    case 128: return F::template run<TS, 128>(args...);                                        \
    default: return F::template run<TS, 256>(args...);                                         \
    }
    switch (dtype) {
    case QKN_BF16: QKN_BY_D(__nv_bfloat16)
    case QKN_FP32: QKN_BY_D(float)
    case QKN_FP16: QKN_BY_D(__half)
    default: QKN_BY_D(__nv_fp8_e4m3)
    }
#undef QKN_BY_D
}

struct PerHead {
    template <typename TS, int D, typename... A>
    static int run(A... a) { return launch_per_head<TS, D>(a...); }
};
struct Layerwise {
    template <typename TS, int D, typename... A>
    static int run(A... a) { return launch_layerwise<TS, D, kFused>(a...); }
};
struct LayerwisePartials {
    template <typename TS, int D, typename... A>
    static int run(A... a) { return launch_layerwise<TS, D, kPartials>(a...); }
};
struct LayerwiseApply {
    template <typename TS, int D, typename... A>
    static int run(A... a) { return launch_layerwise<TS, D, kApply>(a...); }
};

}  // namespace


// ------------------------------------------- entry point without allocation --
// Library-owned scratch for qknorm_layerwise_noalloc: the per-token partial
// sums (two fp32 per token) that the two tensor-parallel steps pass between
// them.  Every GPU that loads the library holds this array until the process
// exits.  Host code must not use the symbol's address directly: on the host
// it names a stand-in, not device memory, so the device address is looked up
// once per device with cudaGetSymbolAddress.
constexpr int64_t kNoAllocMaxTokens = 65536;  // 512 KiB of partial sums
static __device__ __align__(256) float g_noalloc_partials[2 * kNoAllocMaxTokens];

namespace {
std::mutex g_noalloc_mu;
float *g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_partials on the current device; the first call
// on a device looks it up (with that device current).
int noalloc_scratch(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return QKN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_partials);
        if (e != cudaSuccess) return cuda_fail(e);
        g_noalloc_ptr[dev] = static_cast<float *>(p);
    }
    *out = g_noalloc_ptr[dev];
    return QKN_OK;
}
}  // namespace

extern "C" {

int qknorm_per_head(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
                    const float *gamma_q, const float *gamma_k, float eps, void *stream)
{
    bool done = false;
    const int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, &done);
    if (rc != QKN_OK || done) return rc;
    return dispatch<PerHead>(dtype, D, qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps,
                             static_cast<cudaStream_t>(stream));
}

int qknorm_layerwise(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
                     const float *gamma_q, const float *gamma_k, float eps, int nshards,
                     void *stream)
{
    bool done = false;
    const int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, &done);
    if (rc != QKN_OK) return rc;
    if (nshards != 1 && nshards != 2 && nshards != 4 && nshards != 8) return QKN_ERR_NSHARDS;
    if (Hq % nshards != 0 || Hk % nshards != 0) return QKN_ERR_NSHARDS;
    if (done) return QKN_OK;
    return dispatch<Layerwise>(dtype, D, qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps,
                               nshards, static_cast<cudaStream_t>(stream));
}

int qknorm_layerwise_partials(const void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                              int64_t row_stride, float *partials, void *stream)
{
    bool done = false;
    // The weights play no part here; validate the buffer as if they were set.
    const float *no_gamma = reinterpret_cast<const float *>(qkv);
    int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, Hq > 0 ? no_gamma : nullptr,
                      Hk > 0 ? no_gamma : nullptr, 0.f, &done);
    if (rc != QKN_OK || done) return rc;
    if (partials == nullptr) return QKN_ERR_NULL;
    if (((uintptr_t)partials & 7u) != 0) return QKN_ERR_ALIGN;
    return dispatch<LayerwisePartials>(dtype, D, const_cast<void *>(qkv), T, Hq, Hk, row_stride,
                                       (const float *)nullptr, (const float *)nullptr, 0.f, 1,
                                       static_cast<cudaStream_t>(stream), -1.f, -1.f, partials);
}

int qknorm_layerwise_apply(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                           int64_t row_stride, const float *gamma_q, const float *gamma_k,
                           const float *sums, int64_t len_q, int64_t len_k, float eps,
                           void *stream)
{
    bool done = false;
    const int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, &done);
    if (rc != QKN_OK) return rc;
    if ((Hq > 0 && len_q < (int64_t)Hq * D) || (Hk > 0 && len_k < (int64_t)Hk * D) ||
        len_q > (1 << 24) || len_k > (1 << 24))
        return QKN_ERR_SHAPE;
    if (done) return QKN_OK;
    if (sums == nullptr) return QKN_ERR_NULL;
    if (((uintptr_t)sums & 7u) != 0) return QKN_ERR_ALIGN;
    return dispatch<LayerwiseApply>(dtype, D, qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps,
                                    1, static_cast<cudaStream_t>(stream), (float)len_q,
                                    (float)len_k, const_cast<float *>(sums));
}

int qknorm_layerwise_noalloc(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D,
                             int64_t row_stride, const float *gamma_q, const float *gamma_k,
                             float eps, void *stream)
{
    bool done = false;
    int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, &done);
    if (rc != QKN_OK) return rc;
    if (T > kNoAllocMaxTokens) return QKN_ERR_TOO_LARGE;
    if (done) return QKN_OK;
    float *scratch = nullptr;
    if ((rc = noalloc_scratch(&scratch)) != QKN_OK) return rc;
    // Every entry the second step reads is written by the first step of this
    // call, so the scratch needs no clearing.
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    rc = dispatch<LayerwisePartials>(dtype, D, qkv, T, Hq, Hk, row_stride, (const float *)nullptr,
                                     (const float *)nullptr, 0.f, 1, s, -1.f, -1.f, scratch);
    if (rc != QKN_OK) return rc;
    return dispatch<LayerwiseApply>(dtype, D, qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps,
                                    1, s, (float)((int64_t)Hq * D), (float)((int64_t)Hk * D),
                                    scratch);
}

const char *qknorm_status_string(int status)
{
    switch (status) {
    case QKN_OK: return "ok";
    case QKN_ERR_NULL: return "a required pointer is NULL";
    case QKN_ERR_SHAPE: return "invalid shape (negative size, no heads, or row_stride < (Hq+2*Hk)*D)";
    case QKN_ERR_ALIGN: return "qkv, gamma or row_stride bytes not 16-byte aligned";
    case QKN_ERR_NSHARDS: return "nshards must be 1, 2, 4 or 8 and divide Hq and Hk";
    case QKN_ERR_UNSUPPORTED: return "unsupported dtype, head_dim, or token span too wide for one block";
    case QKN_ERR_CUDA: return "CUDA runtime error (see qknorm_last_cuda_error)";
    case QKN_ERR_EPS: return "eps must be finite and >= 0";
    case QKN_ERR_TOO_LARGE:
        return "T exceeds the 65536 tokens of qknorm_layerwise_noalloc's static scratch";
    default: return "unknown status";
    }
}

int qknorm_last_cuda_error(void) { return g_last_cuda_error; }

int qknorm_wait_timeouts(unsigned int *count)
{
    if (count == nullptr) return QKN_ERR_NULL;
    const cudaError_t e = cudaMemcpyFromSymbol(count, g_wait_timeouts, sizeof(unsigned int));
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

int qknorm_version(void) { return 103; }

}  // extern "C"
