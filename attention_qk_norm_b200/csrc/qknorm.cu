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
// (token, head) row of D elements.  Each lane holds D*sizeof/16/LPR 16-byte
// vectors of the row, sums squares in fp32, and the sub-warp reduces with
// xor shuffles.  Every thread keeps U rows in flight per iteration and its
// slice of gamma_q / gamma_k in registers for the whole launch.
//
// Layerwise (SwiftQK abstract; review key_machinery): one thread block owns
// a token at a time (persistent, grid-stride over tokens).  Each head's
// partial sum of squares goes to shared memory; per vector (q, k), one warp
// forms each emulated shard's fp32 partial from its own heads only, stores
// the n shard scalars to shared memory (the scalar exchange), and combines
// them; then every thread scales its registers by the vector's inverse RMS.
// The next token's data is loaded before the current token's reduction so
// that the loads overlap the barriers.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <math.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "qknorm.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxShards = 8;

// ---------------------------------------------------------------- vectors --
template <typename TS>
struct Storage;

template <>
struct Storage<__nv_bfloat16> {
    static constexpr int kVec = 8;  // elements per 16-byte vector
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

// Streaming (evict-first) 16-byte accesses: each element is touched once.
__device__ __forceinline__ uint4 load_stream(const uint4 *p) { return __ldcs(p); }
__device__ __forceinline__ void store_stream(uint4 *p, const uint4 &v) { __stcs(p, v); }

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

// ---------------------------------------------------------------- per-head --
constexpr int kPerHeadThreads = 256;

template <typename TS, int D, int U>
__global__ void __launch_bounds__(kPerHeadThreads)
qkn_per_head_kernel(TS *__restrict__ qkv, int64_t row_stride, uint64_t rows, uint32_t heads,
                    uint32_t Hq, const float *__restrict__ gamma_q,
                    const float *__restrict__ gamma_k, float eps)
{
    using S = Storage<TS>;
    constexpr int kVec = S::kVec;
    constexpr int kNV = D / kVec;                  // 16-byte vectors per row
    constexpr int kLPR = kNV < 32 ? kNV : 32;      // lanes per row
    constexpr int kVPL = kNV / kLPR;               // vectors per lane per row
    constexpr int kEPL = kVPL * kVec;              // elements per lane per row
    static_assert(32 % kLPR == 0 && kNV % kLPR == 0, "row must map onto a sub-warp");

    const uint64_t tid = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const uint32_t lane = (uint32_t)(tid % kLPR);
    const uint64_t group = tid / kLPR;
    const uint64_t ngroups = ((uint64_t)gridDim.x * blockDim.x) / kLPR;

    // This lane's columns are fixed: vectors lane, lane + LPR, ... of a row.
    float gq[kEPL], gk[kEPL];
#pragma unroll
    for (int v = 0; v < kVPL; ++v) {
        const int col = (lane + v * kLPR) * kVec;
        float tq[kVec], tk[kVec];
        load_gamma<kVec>(gamma_q + col, tq);
        if (gamma_k != nullptr) load_gamma<kVec>(gamma_k + col, tk);
#pragma unroll
        for (int e = 0; e < kVec; ++e) {
            gq[v * kVec + e] = tq[e];
            gk[v * kVec + e] = gamma_k != nullptr ? tk[e] : tq[e];
        }
    }

    const bool small = rows <= 0xffffffffull;
    const uint64_t step = ngroups * U;
    // The trip count is the same for every thread, so whole warps reach each
    // shuffle together; rows past the end contribute zeros and store nothing.
    for (uint64_t base = 0; base < rows; base += step) {
        uint4 x[U][kVPL];
        uint4 *ptr[U];
        bool is_q[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
            const uint64_t r = base + (uint64_t)k * ngroups + group;
            ptr[k] = nullptr;
            is_q[k] = true;
            if (r < rows) {
                uint64_t t, h;
                if (small) {
                    const uint32_t r32 = (uint32_t)r;
                    t = r32 / heads;
                    h = r32 - (uint32_t)t * heads;
                } else {
                    t = r / heads;
                    h = r - t * heads;
                }
                is_q[k] = h < Hq;
                ptr[k] = reinterpret_cast<uint4 *>(qkv + (int64_t)t * row_stride + (int64_t)h * D);
#pragma unroll
                for (int v = 0; v < kVPL; ++v) x[k][v] = load_stream(ptr[k] + lane + v * kLPR);
            } else {
#pragma unroll
                for (int v = 0; v < kVPL; ++v) x[k][v] = make_uint4(0u, 0u, 0u, 0u);
            }
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
            if (ptr[k] != nullptr) {
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    float o[kVec];
#pragma unroll
                    for (int e = 0; e < kVec; ++e) {
                        const float g = is_q[k] ? gq[v * kVec + e] : gk[v * kVec + e];
                        o[e] = f[v][e] * rinv * g;
                    }
                    store_stream(ptr[k] + lane + v * kLPR, S::pack(o));
                }
            }
        }
    }
}

// --------------------------------------------------------------- layerwise --
// Shared-memory scratch of one block, laid out after the per-head partials:
//   part[heads]          per-head fp32 partial sums of squares
//   tree[heads]          leaves / partial sums of the fixed reduction tree
//   shard[2][8]          the emulated ranks' scalar partials (q, k)
//   rinv[2]              inverse RMS of the q and k vectors
struct LayerwiseSmem {
    float *part, *tree, *shard, *rinv;
    __device__ LayerwiseSmem(float *base, int heads)
        : part(base), tree(base + heads), shard(base + 2 * heads),
          rinv(base + 2 * heads + 2 * kMaxShards) {}
};

// One warp: inverse RMS of one vector of `nh` heads from their partials.
//
// The reduction tree is fixed by nh alone: nh = m * 2^k with m odd; leaf i
// is the in-order sum of heads [i*m, (i+1)*m), and the 2^k leaves are summed
// pairwise (adjacent pairs first).  A shard of nh/n heads (n a power of two
// dividing nh) is then exactly one subtree, so its partial S_r is formed from
// its own heads only; the n scalars are written to shared memory and combined
// pairwise, which finishes the same tree.  Hence the result does not depend
// on n, bit for bit.
__device__ __forceinline__ void combine_vector(const float *part, float *tree, float *shard,
                                               float *rinv_out, int nh, int nshards,
                                               float len, float eps, int lane)
{
    if (nh == 0) return;
    int m = nh;
    while ((m & 1) == 0) m >>= 1;
    const int leaves = nh / m;
    for (int i = lane; i < leaves; i += 32) {
        float s = 0.f;
        for (int j = 0; j < m; ++j) s += part[i * m + j];
        tree[i] = s;
    }
    __syncwarp();
    const int per_shard = leaves / nshards;  // leaves in one shard's subtree
    for (int w = 1; w < per_shard; w *= 2) {
        for (int i = lane * 2 * w; i < leaves; i += 64 * w) tree[i] += tree[i + w];
        __syncwarp();
    }
    // Scalar exchange: shard r publishes S_r; the combine reads only these.
    if (lane < nshards) shard[lane] = tree[lane * per_shard];
    __syncwarp();
    if (lane == 0) {
        float s[kMaxShards];
        for (int r = 0; r < nshards; ++r) s[r] = shard[r];
        for (int w = 1; w < nshards; w *= 2)
            for (int r = 0; r < nshards; r += 2 * w) s[r] += s[r + w];
        *rinv_out = rsqrtf(s[0] / len + eps);
    }
}

// Block-size ceiling by elements per thread, so that one token's block fits
// the 64K-register file without spills.  With gamma held in registers:
// 1024 threads up to 8 elements, 768 at 16, 512 at 32.  The variant that
// reads gamma from L1 at scale time keeps fewer registers: 1024 up to 16
// elements, 768 at 32.
constexpr int layerwise_max_threads(int ept, bool gamma_regs)
{
    return gamma_regs ? (ept <= 8 ? 1024 : (ept <= 16 ? 768 : 512)) : (ept <= 16 ? 1024 : 768);
}

template <typename TS, int D, int VPT, bool kGammaRegs>
__global__ void __launch_bounds__(layerwise_max_threads(VPT * Storage<TS>::kVec, kGammaRegs))
qkn_layerwise_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, int Hq,
                                     int Hk, int nshards, const float *__restrict__ gamma_q,
                                     const float *__restrict__ gamma_k, float eps, float len_q,
                                     float len_k)
{
    using S = Storage<TS>;
    constexpr int kVec = S::kVec;
    constexpr int kNV = D / kVec;    // 16-byte vectors per head
    constexpr int kLPH = kNV / VPT;  // threads per head
    constexpr int kEPT = VPT * kVec; // elements per thread
    static_assert(kNV % VPT == 0 && 32 % kLPH == 0, "head must map onto a sub-warp");

    extern __shared__ float smem_raw[];
    const int heads = Hq + Hk;
    LayerwiseSmem sm(smem_raw, heads);

    const int h = threadIdx.x / kLPH;
    const int l = threadIdx.x % kLPH;
    const bool active = h < heads;
    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    const int nwarps = blockDim.x / 32;

    // Fixed columns of this thread: vectors l, l + LPH, ... of head h.
    const float *gb = !active ? gamma_q
                      : (h < Hq ? gamma_q + (int64_t)h * D : gamma_k + (int64_t)(h - Hq) * D);
    float g[kGammaRegs ? kEPT : 1];
#pragma unroll
    for (int e = 0; e < (kGammaRegs ? kEPT : 1); ++e) g[e] = 0.f;
    if (kGammaRegs && active) {
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            float t4[kVec];
            load_gamma<kVec>(gb + (l + v * kLPH) * kVec, t4);
#pragma unroll
            for (int e = 0; e < kVec; ++e) g[v * kVec + e] = t4[e];
        }
    }
    const int64_t col0 = (int64_t)h * D;

    uint4 cur[VPT], nxt[VPT];
#pragma unroll
    for (int v = 0; v < VPT; ++v) cur[v] = nxt[v] = make_uint4(0u, 0u, 0u, 0u);
    int64_t t = blockIdx.x;
    if (active && t < T) {
        const uint4 *p = reinterpret_cast<const uint4 *>(qkv + t * row_stride + col0);
#pragma unroll
        for (int v = 0; v < VPT; ++v) cur[v] = load_stream(p + l + v * kLPH);
    }
    for (; t < T; t += gridDim.x) {
        const int64_t tn = t + gridDim.x;
        if (active && tn < T) {
            const uint4 *p = reinterpret_cast<const uint4 *>(qkv + tn * row_stride + col0);
#pragma unroll
            for (int v = 0; v < VPT; ++v) nxt[v] = load_stream(p + l + v * kLPH);
        }
        float f[VPT][kVec];
        float s = 0.f;
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            S::unpack(cur[v], f[v]);
#pragma unroll
            for (int e = 0; e < kVec; ++e) s = fmaf(f[v][e], f[v][e], s);
        }
        s = group_sum<kLPH>(s);
        if (active && l == 0) sm.part[h] = s;
        __syncthreads();
        if (warp == 0)
            combine_vector(sm.part, sm.tree, sm.shard, sm.rinv, Hq, nshards, len_q, eps, lane);
        if (warp == (nwarps > 1 ? 1 : 0))
            combine_vector(sm.part + Hq, sm.tree + Hq, sm.shard + kMaxShards, sm.rinv + 1, Hk,
                           nshards, len_k, eps, lane);
        __syncthreads();
        if (active) {
            const float rinv = sm.rinv[h < Hq ? 0 : 1];
            uint4 *p = reinterpret_cast<uint4 *>(qkv + t * row_stride + col0);
#pragma unroll
            for (int v = 0; v < VPT; ++v) {
                float o[kVec], gv[kVec];
                if constexpr (kGammaRegs) {
#pragma unroll
                    for (int e = 0; e < kVec; ++e) gv[e] = g[v * kVec + e];
                } else {
                    load_gamma<kVec>(gb + (l + v * kLPH) * kVec, gv);
                }
#pragma unroll
                for (int e = 0; e < kVec; ++e) o[e] = f[v][e] * rinv * gv[e];
                store_stream(p + l + v * kLPH, S::pack(o));
            }
        }
#pragma unroll
        for (int v = 0; v < VPT; ++v) cur[v] = nxt[v];
    }
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
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

int device_sms(int *sms)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev < 0 || dev >= kMaxDevices) return QKN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (g_dev[dev].sms == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e);
        g_dev[dev].sms = n;
    }
    *sms = g_dev[dev].sms;
    return QKN_OK;
}

// Resident blocks per SM of one kernel at one block size (cached).
template <typename Kernel>
int blocks_per_sm(Kernel k, int threads, size_t smem, int *out)
{
    int n = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem);
    if (e != cudaSuccess) return cuda_fail(e);
    *out = n > 0 ? n : 1;
    return QKN_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

int elem_size(int dtype) { return dtype == QKN_BF16 ? 2 : (dtype == QKN_FP32 ? 4 : 0); }

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

constexpr int kPerHeadRowsInFlight = 2;

template <typename TS, int D>
int launch_per_head(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride, const float *gq,
                    const float *gk, float eps, cudaStream_t stream)
{
    constexpr int U = kPerHeadRowsInFlight;
    constexpr int kNV = D / Storage<TS>::kVec;
    constexpr int kLPR = kNV < 32 ? kNV : 32;
    auto kern = qkn_per_head_kernel<TS, D, U>;
    int sms = 0, per_sm = 0, rc;
    if ((rc = device_sms(&sms)) != QKN_OK) return rc;
    static std::atomic<int> cached_per_sm{0};  // same sm_100a image on every device
    per_sm = cached_per_sm.load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if ((rc = blocks_per_sm(kern, kPerHeadThreads, 0, &per_sm)) != QKN_OK) return rc;
        cached_per_sm.store(per_sm, std::memory_order_relaxed);
    }
    // Qwen3 gamma is shared by every head: pass nullptr for K when Hk == 0.
    const float *gq_eff = Hq > 0 ? gq : gk;
    const float *gk_eff = Hk > 0 ? gk : nullptr;
    const uint64_t rows = (uint64_t)T * (uint64_t)(Hq + Hk);
    const uint64_t rows_per_block = (uint64_t)(kPerHeadThreads / kLPR) * U;
    const uint64_t need = (rows + rows_per_block - 1) / rows_per_block;
    const uint64_t cap = (uint64_t)sms * per_sm;
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    kern<<<grid, kPerHeadThreads, 0, stream>>>(static_cast<TS *>(qkv), row_stride, rows,
                                               (uint32_t)(Hq + Hk), (uint32_t)Hq, gq_eff, gk_eff,
                                               eps);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

// A layerwise kernel variant exists when a head splits into whole 16-byte
// vectors per thread on at most 32 lanes, with at most 32 elements per thread.
template <typename TS, int D, int VPT>
constexpr bool layerwise_vpt_ok()
{
    constexpr int kNV = D / Storage<TS>::kVec;
    return kNV % VPT == 0 && kNV / VPT <= 32 && VPT * Storage<TS>::kVec <= 32;
}

template <typename TS, int D, int VPT>
int launch_layerwise_vpt(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride,
                         const float *gq, const float *gk, float eps, int nshards, int threads,
                         cudaStream_t stream)
{
    const int heads = Hq + Hk;
    constexpr int kEPT = VPT * Storage<TS>::kVec;
    // Gamma in registers when the block fits that variant, else from L1.
    auto kern = threads <= layerwise_max_threads(kEPT, true)
                    ? qkn_layerwise_kernel<TS, D, VPT, true>
                    : qkn_layerwise_kernel<TS, D, VPT, false>;
    const bool regs_variant = threads <= layerwise_max_threads(kEPT, true);
    const size_t smem = (size_t)(2 * heads + 2 * kMaxShards + 2) * sizeof(float);
    int sms = 0, per_sm = 0, rc;
    if ((rc = device_sms(&sms)) != QKN_OK) return rc;
    // Per block size (a multiple of 32 up to 1024): the register-limited
    // maximum and the resident blocks per SM, both computed once.
    static std::atomic<int> max_threads[2];
    static std::atomic<int> cached[2][33];
    int mt = max_threads[regs_variant].load(std::memory_order_relaxed);
    if (mt == 0) {
        cudaFuncAttributes attr;
        const cudaError_t e = cudaFuncGetAttributes(&attr, kern);
        if (e != cudaSuccess) return cuda_fail(e);
        mt = attr.maxThreadsPerBlock;
        max_threads[regs_variant].store(mt, std::memory_order_relaxed);
    }
    if (threads > mt) return QKN_ERR_UNSUPPORTED;
    per_sm = cached[regs_variant][threads / 32].load(std::memory_order_relaxed);
    if (per_sm == 0) {
        if ((rc = blocks_per_sm(kern, threads, smem, &per_sm)) != QKN_OK) return rc;
        cached[regs_variant][threads / 32].store(per_sm, std::memory_order_relaxed);
    }
    const int64_t cap = (int64_t)sms * per_sm;
    const unsigned grid = (unsigned)(T < cap ? T : cap);
    const float len_q = (float)((int64_t)Hq * D);  // exact: spans are < 2^24 elements
    const float len_k = (float)((int64_t)Hk * D);
    kern<<<grid, threads, smem, stream>>>(static_cast<TS *>(qkv), row_stride, T, Hq, Hk, nshards,
                                          gq, gk, eps, len_q, len_k);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

// Vectors per thread: the fewest that keep a token's block within
// kLayerwiseTargetThreads, else within 1024 threads; at most 32 fp32
// elements per thread (registers).
constexpr int kLayerwiseTargetThreads = 256;

template <typename TS, int D>
int launch_layerwise(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride, const float *gq,
                     const float *gk, float eps, int nshards, cudaStream_t stream)
{
    constexpr int kNV = D / Storage<TS>::kVec;
    constexpr int kMaxVPT = 32 / Storage<TS>::kVec;  // 4 for bf16, 8 for fp32
    const int64_t heads = Hq + Hk;
    int chosen = 0;
    for (int pass = 0; pass < 2 && chosen == 0; ++pass) {
        const int64_t limit = pass == 0 ? kLayerwiseTargetThreads : 768;
        for (int vpt = 1; vpt <= kMaxVPT; vpt *= 2) {
            if (kNV % vpt != 0 || kNV / vpt > 32) continue;  // mirrors layerwise_vpt_ok
            const int64_t threads = ((heads * (kNV / vpt) + 31) / 32) * 32;
            if (threads <= limit) {
                chosen = vpt;
                break;
            }
        }
    }
    if (chosen == 0) return QKN_ERR_UNSUPPORTED;
    const int threads = (int)(((heads * (kNV / chosen) + 31) / 32) * 32);
    switch (chosen) {
    case 1:
        if constexpr (layerwise_vpt_ok<TS, D, 1>())
            return launch_layerwise_vpt<TS, D, 1>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,
                                                  nshards, threads, stream);
        break;
    case 2:
        if constexpr (layerwise_vpt_ok<TS, D, 2>())
            return launch_layerwise_vpt<TS, D, 2>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,
                                                  nshards, threads, stream);
        break;
    case 4:
        if constexpr (layerwise_vpt_ok<TS, D, 4>())
            return launch_layerwise_vpt<TS, D, 4>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,
                                                  nshards, threads, stream);
        break;
    case 8:
        if constexpr (layerwise_vpt_ok<TS, D, 8>())
            return launch_layerwise_vpt<TS, D, 8>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,
                                                  nshards, threads, stream);
        break;
    default:
        break;
    }
    return QKN_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" {

int qknorm_per_head(void *qkv, int dtype, int64_t T, int Hq, int Hk, int D, int64_t row_stride,
                    const float *gamma_q, const float *gamma_k, float eps, void *stream)
{
    bool done = false;
    const int rc = validate(qkv, dtype, T, Hq, Hk, D, row_stride, gamma_q, gamma_k, eps, &done);
    if (rc != QKN_OK || done) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QKN_BF16) {
        switch (D) {
        case 64: return launch_per_head<__nv_bfloat16, 64>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
        case 128: return launch_per_head<__nv_bfloat16, 128>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
        default: return launch_per_head<__nv_bfloat16, 256>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
        }
    }
    switch (D) {
    case 64: return launch_per_head<float, 64>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
    case 128: return launch_per_head<float, 128>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
    default: return launch_per_head<float, 256>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, s);
    }
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
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == QKN_BF16) {
        switch (D) {
        case 64: return launch_layerwise<__nv_bfloat16, 64>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
        case 128: return launch_layerwise<__nv_bfloat16, 128>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
        default: return launch_layerwise<__nv_bfloat16, 256>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
        }
    }
    switch (D) {
    case 64: return launch_layerwise<float, 64>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
    case 128: return launch_layerwise<float, 128>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
    default: return launch_layerwise<float, 256>(qkv, T, Hq, Hk, row_stride, gamma_q, gamma_k, eps, nshards, s);
    }
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
    default: return "unknown status";
    }
}

int qknorm_last_cuda_error(void) { return g_last_cuda_error; }

int qknorm_version(void) { return 100; }

}  // extern "C"
