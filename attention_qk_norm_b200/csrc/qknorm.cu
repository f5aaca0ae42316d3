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
// (or thread-block cluster, for tokens too wide for one block) walks tokens
// with a grid stride.  Each thread copies its vectors of the next token (the
// next two for FP8 on long inputs) into a shared-memory ring with cp.async
// while it works on the current one (at decode sizes it loads them straight
// into registers instead).  The
// per-head partial sums of squares meet in shared memory behind one barrier
// (across a cluster, on transaction barriers); then each warp, for the
// vectors (q, k) its threads hold, forms every emulated shard's fp32 partial
// from that shard's heads alone and combines the shard scalars, and every
// thread scales its vectors by the inverse RMS of its vector.
//
// Both kernels are launched with programmatic dependent launch: they wait on
// griddepcontrol.wait before their first load or store, so a kernel earlier
// in the stream always finishes first, and they allow the next kernel to be
// scheduled as soon as all of their blocks are resident.  Before the wait a
// block only computes its first rows' addresses and prefetches those rows
// into L2 (prefetch_l2), which overlaps the latency of its first loads with
// the draining of the grid before it.  The
// only wait between blocks is inside a thread-block cluster of the layerwise
// kernel, whose blocks the hardware schedules together; each such wait gives
// up after a time limit, so no kernel here can hang.
//
// Files: storage.cuh (vectors and device helpers), per_head.cuh and
// layerwise.cuh (the kernels), and this file (launch shapes and the C ABI).
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

#include "layerwise.cuh"
#include "per_head.cuh"
#include "storage.cuh"
#include "tp_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;

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
    constexpr int U = per_head_rows_in_flight<TS>();
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

template <typename TS, int D, int VPT, bool kCluster, int kMode, int kSched = kSchedRing>
int launch_layerwise_vpt(void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride,
                         const float *gq, const float *gk, float eps, int threads, int cluster,
                         float inv_len_q, float inv_len_k, SumPlan plan_q, SumPlan plan_k,
                         float *aux, cudaStream_t stream)
{
    auto kern = [] {
        if constexpr (layerwise_gamma_regs<TS, VPT>())
            return qkn_layerwise_kernel<TS, D, VPT, kCluster, kMode, kSched>;
        else
            return qkn_layerwise_l1_kernel<TS, D, VPT, kMode>;
    }();
    static KernelCache kc;
    const int heads = Hq + Hk;
    const size_t span = (size_t)(heads / cluster) * D * sizeof(TS);
    const size_t stages = layerwise_stages<TS, kSched>();
    const size_t smem = stages * span + (size_t)2 * heads * sizeof(float) + 2 * sizeof(uint64_t);
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

// Storage types whose large fused launches use the overlap schedule.
template <typename TS>
constexpr bool layerwise_overlap_type()
{
    return Storage<TS>::kVec == 4 || Storage<TS>::kVec == 16;  // fp32, FP8
}

// The kernel instance for one vectors-per-thread count: the schedule (only
// fused launches use the direct and overlap ones, and the overlap only for
// fp32 and FP8) and whether the launch is a cluster.  Gamma-through-L1
// launches are single blocks on the ring.
template <typename TS, int D, int V, int kMode>
int launch_layerwise_sched(int sched, void *qkv, int64_t T, int Hq, int Hk, int64_t row_stride,
                           const float *gq, const float *gk, float eps, int threads, int cluster,
                           float inv_len_q, float inv_len_k, SumPlan plan_q, SumPlan plan_k,
                           float *aux, cudaStream_t stream)
{
#define QKN_LW_LAUNCH(CL, SCHED)                                                               \
    launch_layerwise_vpt<TS, D, V, CL, kMode, SCHED>(qkv, T, Hq, Hk, row_stride, gq, gk, eps,  \
                                                     threads, CL ? cluster : 1, inv_len_q,     \
                                                     inv_len_k, plan_q, plan_k, aux, stream)
    if constexpr (layerwise_gamma_regs<TS, V>()) {
        if constexpr (kMode == kFused) {
            if (sched == kSchedDirect)
                return cluster > 1 ? QKN_LW_LAUNCH(true, kSchedDirect)
                                   : QKN_LW_LAUNCH(false, kSchedDirect);
            if constexpr (layerwise_overlap_type<TS>()) {
                if (sched == kSchedOverlap)
                    return cluster > 1 ? QKN_LW_LAUNCH(true, kSchedOverlap)
                                       : QKN_LW_LAUNCH(false, kSchedOverlap);
            }
        }
        if (cluster > 1) return QKN_LW_LAUNCH(true, kSchedRing);
    }
    return QKN_LW_LAUNCH(false, kSchedRing);
#undef QKN_LW_LAUNCH
}

// Launch shape, chosen from measurements on B200 over the four storage types,
// head_dim 64 to 256 and 40 to 72 heads:
//  * the smallest cluster size CL (1, 2, 4 or 8 blocks, dividing the head
//    count) for which some vectors-per-thread count VPT keeps gamma in
//    registers (VPT * kVec <= 32) and the block within 576 threads;
//  * the fewest such VPT, but at least 2: with one vector per thread the
//    per-token work of a thread is too short for its fixed per-token cost;
//  * on inputs of at most one block per SM (T times CL up to the SM count),
//    that VPT with the direct schedule for fused launches: each block has one
//    token, so there is nothing to prefetch and no ring;
//  * on other short inputs, fewer than 12 tokens per resident cluster, twice
//    that VPT when gamma still fits: half the threads per block, about twice
//    the resident blocks, so more tokens are under way at once.
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
    SumPlan p = {0, 0, 0, 0};
    if (nh > 0) {
        const int p2 = nh & (-nh);
        p.used = p2 < 32 ? p2 : 32;
        p.per_lane = nh / p.used;
        p.per_shard = p.used / nshards;  // nshards is a power of two dividing nh
    }
    return p;
}

// The warp tree of a plain fused launch whose warps each hold hpw heads:
// used when each vector's head count is a power of two up to 64, no warp
// holds heads of both vectors, and each vector spans at most 8 warps.
void set_warp_tree(SumPlan &plan_q, SumPlan &plan_k, int Hq, int Hk, int hpw)
{
    auto binary = [](int nh) { return nh > 0 && (nh & (nh - 1)) == 0 && nh <= 64; };
    const int nq = Hq / hpw, nk = Hk > 0 ? (Hk + hpw - 1) / hpw : 0;
    if ((Hq == 0 || (binary(Hq) && Hq % hpw == 0)) && (Hk == 0 || binary(Hk)) && nq <= 8 &&
        nk <= 8) {
        plan_q.warps = nq;
        plan_k.warps = nk;
    }
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
    SumPlan plan_q = sum_plan(Hq, nshards), plan_k = sum_plan(Hk, nshards);
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
    int sched = kSchedRing;
    bool short_launch = false;  // the direct schedule, or twice the VPT
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
        // The vectors per thread depend on the shape and T only, never on the
        // mode, so the tensor-parallel steps sum exactly as the fused kernel.
        bool doubled = false;
        if (T * cluster <= info.sms) {
            // At most one block per SM, each with one token: nothing to
            // prefetch (measured on B200: T=1..64 gain 11-22%; at T=256, with
            // SMs shared, the ring with twice the VPT is 7% faster).
            if (kMode == kFused) sched = kSchedDirect;
        } else if (can_double &&
                   T < kLayerwiseShortTokens * pipelines(layerwise_regs(ept, false, kVec))) {
            chosen *= 2;
            doubled = true;
        }
        if (!doubled && kMode == kFused && layerwise_overlap_type<TS>() && sched == kSchedRing &&
            T >= kLayerwiseShortTokens * pipelines(layerwise_regs(ept, true, kVec)))
            sched = kSchedOverlap;
        short_launch = doubled || sched == kSchedDirect;
    }
    for (int vpt = 1; vpt <= kNV && chosen == 0; vpt *= 2)
        if (vpt_ok(vpt) && threads_for(1, vpt) <= 1024) chosen = vpt;
    if (chosen == 0) return QKN_ERR_UNSUPPORTED;
    const int threads = (int)(((heads / cluster * (kNV / chosen)) + 31) / 32 * 32);
    // The warp tree, where it applies, for FP8 and for short inputs: measured
    // on B200 it gains 3-5% for FP8 (32q/8kv and 64q/8kv, T = 8192 to 32768)
    // and 1-2% on short bf16 inputs (T = 256 to 4096), where the chain after
    // the barrier is a larger part of a token's time; on long bf16 / fp16
    // inputs the per-head partials measured 1% faster.
    if (kMode == kFused && cluster == 1 && chosen * kVec <= 32 && (kVec == 16 || short_launch))
        set_warp_tree(plan_q, plan_k, Hq, Hk, 32 / (kNV / chosen));
#define QKN_LW_CASE(V)                                                                         \
    case V:                                                                                    \
        if constexpr (layerwise_vpt_ok<TS, D, V>())                                            \
            return launch_layerwise_sched<TS, D, V, kMode>(sched, qkv, T, Hq, Hk, row_stride,   \
                                                           gq, gk, eps, threads, cluster,      \
                                                           inv_len_q, inv_len_k, plan_q,       \
                                                           plan_k, aux, stream);               \
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

// ---------------------------------------- tensor-parallel exchange, P2P --
// Launch shape of the in-kernel exchange (tp_kernel.cuh): one block per
// token (no cluster), gamma in registers, the fewest vectors per thread (at
// least 2) within 576 threads.
template <typename TS, int D, int VPT>
int launch_tp_vpt(const TPRankPtrs &ptrs, int nlocal, int64_t T, int Hq, int Hk,
                  int64_t row_stride, float eps, float inv_len_q, float inv_len_k, SumPlan plan_q,
                  SumPlan plan_k, const P2PArgs &p2p, int threads, cudaStream_t stream)
{
    auto kern = qkn_layerwise_tp_kernel<TS, D, VPT>;
    static KernelCache kc;
    const int heads = Hq + Hk;
    const size_t span = (size_t)heads * D * sizeof(TS);
    const size_t smem = kTPStages * span + (size_t)2 * heads * sizeof(float);
    int dev = 0, per_sm = 0, rc;
    DeviceInfo info;
    if ((rc = device_info(&dev, &info)) != QKN_OK) return rc;
    if (smem > (size_t)info.smem_optin) return QKN_ERR_UNSUPPORTED;
    if ((rc = resident_blocks(kern, kc, dev, info, threads, smem, &per_sm)) != QKN_OK) return rc;
    // At most as many blocks per rank as fit resident at once.
    const int64_t per_rank = (int64_t)info.sms * per_sm / nlocal;
    if (per_rank < 1) return QKN_ERR_UNSUPPORTED;
    const int64_t blocks = T < per_rank ? T : per_rank;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks, (unsigned)nlocal);
    cfg.blockDim = dim3((unsigned)threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    if (nlocal > 1) {
        // Several ranks in one launch: their blocks wait on one another, so
        // the launch is cooperative (all blocks resident, or it fails).
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
    } else {
        // One rank per GPU: a block waits only on blocks of other GPUs'
        // launches, never on a block of its own launch, so a plain launch
        // with programmatic dependent launch (as the other kernels) will do.
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ptrs, row_stride, T, Hq, Hk, eps, inv_len_q,
                                       inv_len_k, plan_q, plan_k, p2p);
    if (e == cudaSuccess) e = cudaGetLastError();
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

struct LayerwiseTP {
    template <typename TS, int D>
    static int run(const TPRankPtrs &ptrs, int nlocal, int64_t T, int Hq, int Hk,
                   int64_t row_stride, float eps, float len_q, float len_k, const P2PArgs &p2p,
                   cudaStream_t stream)
    {
        constexpr int kVec = Storage<TS>::kVec;
        constexpr int kNV = D / kVec;
        const int heads = Hq + Hk;
        int vpt = 0;
        for (int v = 2; v * kVec <= 32 && vpt == 0; v *= 2)
            if (v <= kNV && kNV % v == 0 && kNV / v <= 32 &&
                (heads * (kNV / v) + 31) / 32 * 32 <= kLayerwiseMaxThreads)
                vpt = v;
        if (vpt == 0) return QKN_ERR_UNSUPPORTED;
        const int threads = (heads * (kNV / vpt) + 31) / 32 * 32;
        const float inv_len_q = Hq > 0 ? 1.0f / len_q : 0.f;
        const float inv_len_k = Hk > 0 ? 1.0f / len_k : 0.f;
        SumPlan plan_q = sum_plan(Hq, 1), plan_k = sum_plan(Hk, 1);
        set_warp_tree(plan_q, plan_k, Hq, Hk, 32 / (kNV / vpt));
#define QKN_TP_CASE(V)                                                                         \
    case V:                                                                                    \
        if constexpr (layerwise_vpt_ok<TS, D, V>() && layerwise_gamma_regs<TS, V>())           \
            return launch_tp_vpt<TS, D, V>(ptrs, nlocal, T, Hq, Hk, row_stride, eps,           \
                                           inv_len_q, inv_len_k, plan_q, plan_k, p2p,          \
                                           threads, stream);                                   \
        break;
        switch (vpt) {
            QKN_TP_CASE(2)
            QKN_TP_CASE(4)
            QKN_TP_CASE(8)
        default:
            break;
        }
#undef QKN_TP_CASE
        return QKN_ERR_UNSUPPORTED;
    }
};

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

// The communicator of qknorm_layerwise_tp_p2p (see include/qknorm.h).
struct qkn_tp_comm {
    int world = 0, rank = 0, nlocal = 0, device = -1;
    int64_t max_tokens = 0;
    uint64_t timeout_ns = 0;
    bool connected = false;
    uint64_t *own[qkn_tp::kMaxWorld] = {};   // buffers this communicator allocated
    uint64_t *recv[qkn_tp::kMaxWorld] = {};  // every rank's buffer, as this device addresses it
    bool opened[qkn_tp::kMaxWorld] = {};     // recv[r] is an IPC mapping to close
    unsigned int *errors = nullptr;          // device counter of waits that gave up
    uint32_t *abort_tag = nullptr;
    uint32_t *seq = nullptr;                 // device: calls made so far (advanced by each launch)
    uint32_t *done = nullptr;                // device: blocks of the running launch that finished
};

namespace {
constexpr size_t kTPTailBytes = 256;  // the counter and the abort tag, after own[0]'s slots

bool tp_world_ok(int world) { return world == 1 || world == 2 || world == 4 || world == 8; }

// Allocate and zero `n` receive buffers on the current device.
int tp_alloc(qkn_tp_comm *c, int n)
{
    const size_t bytes = qkn_tp::buffer_words(c->max_tokens, c->world) * sizeof(uint64_t);
    for (int i = 0; i < n; ++i) {
        void *p = nullptr;
        cudaError_t e = cudaMalloc(&p, bytes + (i == 0 ? kTPTailBytes : 0));
        if (e == cudaSuccess) e = cudaMemset(p, 0, bytes + (i == 0 ? kTPTailBytes : 0));
        if (e != cudaSuccess) {
            if (p != nullptr) cudaFree(p);
            return cuda_fail(e);
        }
        c->own[i] = static_cast<uint64_t *>(p);
    }
    unsigned char *tail = reinterpret_cast<unsigned char *>(c->own[0]) + bytes;
    c->errors = reinterpret_cast<unsigned int *>(tail);
    c->abort_tag = reinterpret_cast<uint32_t *>(tail + 64);
    c->seq = reinterpret_cast<uint32_t *>(tail + 128);
    c->done = reinterpret_cast<uint32_t *>(tail + 192);
    return QKN_OK;
}

void tp_free(qkn_tp_comm *c)
{
    int prev = -1;
    cudaGetDevice(&prev);
    if (c->device >= 0) cudaSetDevice(c->device);
    for (int r = 0; r < qkn_tp::kMaxWorld; ++r)
        if (c->opened[r]) cudaIpcCloseMemHandle(c->recv[r]);
    for (int i = 0; i < qkn_tp::kMaxWorld; ++i)
        if (c->own[i] != nullptr) cudaFree(c->own[i]);
    if (prev >= 0) cudaSetDevice(prev);
    delete c;
}

int tp_create(int world, int rank, int nlocal, int64_t max_tokens, double timeout_s,
              qkn_tp_comm **out)
{
    if (out == nullptr) return QKN_ERR_NULL;
    *out = nullptr;
    if (!tp_world_ok(world) || rank < 0 || rank >= world) return QKN_ERR_NSHARDS;
    if (max_tokens < 1 || max_tokens > (int64_t)1 << 24) return QKN_ERR_SHAPE;
    if (!(timeout_s > 0.0) || timeout_s > 3600.0) return QKN_ERR_SHAPE;
    qkn_tp_comm *c = new qkn_tp_comm;
    c->world = world;
    c->rank = rank;
    c->nlocal = nlocal;
    c->max_tokens = max_tokens;
    c->timeout_ns = (uint64_t)(timeout_s * 1e9);
    cudaError_t e = cudaGetDevice(&c->device);
    if (e != cudaSuccess) {
        delete c;
        return cuda_fail(e);
    }
    const int rc = tp_alloc(c, nlocal);
    if (rc != QKN_OK) {
        tp_free(c);
        return rc;
    }
    *out = c;
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

int qknorm_tp_comm_create(int world, int rank, int64_t max_tokens, double timeout_s,
                          qkn_tp_comm **comm, void *ipc_handle)
{
    if (ipc_handle == nullptr) return QKN_ERR_NULL;
    int rc = tp_create(world, rank, 1, max_tokens, timeout_s, comm);
    if (rc != QKN_OK) return rc;
    qkn_tp_comm *c = *comm;
    c->recv[rank] = c->own[0];
    const cudaError_t e =
        cudaIpcGetMemHandle(static_cast<cudaIpcMemHandle_t *>(ipc_handle), c->own[0]);
    if (e != cudaSuccess) {
        tp_free(c);
        *comm = nullptr;
        return cuda_fail(e);
    }
    if (world == 1) c->connected = true;
    return QKN_OK;
}

int qknorm_tp_comm_connect(qkn_tp_comm *comm, const void *ipc_handles)
{
    if (comm == nullptr || ipc_handles == nullptr) return QKN_ERR_NULL;
    if (comm->nlocal != 1) return QKN_ERR_UNSUPPORTED;
    if (comm->connected) return QKN_OK;
    const cudaIpcMemHandle_t *h = static_cast<const cudaIpcMemHandle_t *>(ipc_handles);
    for (int r = 0; r < comm->world; ++r) {
        if (r == comm->rank) continue;
        void *p = nullptr;
        const cudaError_t e = cudaIpcOpenMemHandle(&p, h[r], cudaIpcMemLazyEnablePeerAccess);
        if (e != cudaSuccess) return cuda_fail(e);
        comm->recv[r] = static_cast<uint64_t *>(p);
        comm->opened[r] = true;
    }
    comm->connected = true;
    return QKN_OK;
}

int qknorm_tp_comm_create_local(int world, int64_t max_tokens, double timeout_s,
                                qkn_tp_comm **comm)
{
    const int rc = tp_create(world, 0, world, max_tokens, timeout_s, comm);
    if (rc != QKN_OK) return rc;
    for (int r = 0; r < world; ++r) (*comm)->recv[r] = (*comm)->own[r];
    (*comm)->connected = true;
    return QKN_OK;
}

int qknorm_tp_comm_destroy(qkn_tp_comm *comm)
{
    if (comm == nullptr) return QKN_ERR_NULL;
    tp_free(comm);
    return QKN_OK;
}

int qknorm_tp_comm_errors(qkn_tp_comm *comm, unsigned int *count)
{
    if (comm == nullptr || count == nullptr) return QKN_ERR_NULL;
    const cudaError_t e = cudaMemcpy(count, comm->errors, sizeof(unsigned int),
                                     cudaMemcpyDeviceToHost);
    return e == cudaSuccess ? QKN_OK : cuda_fail(e);
}

int qknorm_layerwise_tp_p2p(qkn_tp_comm *comm, void *const *qkv, int dtype, int64_t T, int Hq,
                            int Hk, int D, int64_t row_stride, const float *const *gamma_q,
                            const float *const *gamma_k, float eps, void *stream)
{
    if (comm == nullptr || qkv == nullptr || gamma_q == nullptr || gamma_k == nullptr)
        return QKN_ERR_NULL;
    bool done = false;
    for (int i = 0; i < comm->nlocal; ++i) {
        const int rc = validate(qkv[i], dtype, T, Hq, Hk, D, row_stride, gamma_q[i], gamma_k[i],
                                eps, &done);
        if (rc != QKN_OK) return rc;
    }
    if (T > comm->max_tokens) return QKN_ERR_TOO_LARGE;
    if (done) return QKN_OK;
    if (!comm->connected) return QKN_ERR_UNSUPPORTED;
    int dev = -1;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e);
    if (dev != comm->device) return QKN_ERR_UNSUPPORTED;
    TPRankPtrs ptrs = {};
    for (int i = 0; i < comm->nlocal; ++i) {
        ptrs.qkv[i] = qkv[i];
        ptrs.gamma_q[i] = gamma_q[i];
        ptrs.gamma_k[i] = gamma_k[i];
    }
    P2PArgs a = {};
    for (int r = 0; r < comm->world; ++r) a.recv[r] = comm->recv[r];
    a.errors = comm->errors;
    a.abort_tag = comm->abort_tag;
    a.seq = comm->seq;
    a.done = comm->done;
    a.max_tokens = comm->max_tokens;
    a.timeout_ns = comm->timeout_ns;
    a.world = comm->world;
    a.rank = comm->rank;
    const float len_q = (float)((int64_t)Hq * D * comm->world);
    const float len_k = (float)((int64_t)Hk * D * comm->world);
    return dispatch<LayerwiseTP>(dtype, D, ptrs, comm->nlocal, T, Hq, Hk, row_stride, eps, len_q,
                                 len_k, a, static_cast<cudaStream_t>(stream));
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

int qknorm_version(void) { return 105; }

}  // extern "C"
