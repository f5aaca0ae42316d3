// per_head.cuh -- the per-head QK-Norm kernel.
// Part of libqknorm.so; included by qknorm.cu, the library's one translation
// unit.
#pragma once

#include "storage.cuh"

namespace {

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

}  // namespace

// --------------------------------------------------- per-head, bulk-staged --
// The same arithmetic as qkn_per_head_kernel (fp32 sum of squares, sub-warp
// reduction, (x * rinv) * gamma, one rounding), with the loads moved off the
// threads: a producer warp streams chunks of rows into a ring of shared-memory
// stages with cp.async.bulk, completing on each stage's mbarrier, and eight
// consumer warps normalise the staged rows and store them to global memory.
// The bytes in flight per SM are then set by the ring (up to three stages of
// each resident block), not by registers per thread.  Rows are taken in
// (token, head) order; a chunk is kBulkPasses * NG * U consecutive rows (NG
// row groups of LPR lanes, U rows each per pass), copied as one bulk copy per
// token it touches (one in all when rows are contiguous in memory), and packed
// back to back in its stage.
constexpr int kBulkConsumerWarps = 8;
constexpr int kBulkThreads = 32 * (kBulkConsumerWarps + 1);  // plus the producer warp
constexpr int kBulkStages = 4;
constexpr int kBulkRowsInFlight = 2;

template <typename TS, int D>
struct BulkShape {
    static constexpr int kVec = Storage<TS>::kVec;
    static constexpr int kNV = D / kVec;                        // vectors per row
    static constexpr int kLPR = kNV < 32 ? kNV : 32;            // lanes per row
    static constexpr int kRowBytes = D * (int)sizeof(TS);
    static constexpr int kGroups = 32 * kBulkConsumerWarps / kLPR;  // NG
    static constexpr int kPassRows = kGroups * kBulkRowsInFlight;
    // About 24 KB per chunk: three passes of 8 KB, or one of 16 KB or more.
    static constexpr int kPasses = kPassRows * kRowBytes >= 16384 ? 1 : 24576 / (kPassRows * kRowBytes);
    static constexpr int kChunkRows = kPassRows * kPasses;
    static constexpr int kChunkBytes = kChunkRows * kRowBytes;
    static constexpr int kSmemBytes = kBulkStages * kChunkBytes + 2 * kBulkStages * 8;
};

template <typename TS, int D, bool kHasK>
__global__ void __launch_bounds__(kBulkThreads, 2)
qkn_per_head_bulk_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, uint32_t heads,
                         uint32_t Hq, const float *__restrict__ gamma_q,
                         const float *__restrict__ gamma_k, float eps, uint64_t nchunks)
{
    using S = Storage<TS>;
    using V = typename S::Vec;
    using B = BulkShape<TS, D>;
    constexpr int kVec = S::kVec;
    constexpr int kLPR = B::kLPR;
    constexpr int kVPL = B::kNV / kLPR;  // vectors per lane per row
    constexpr int kEPL = kVPL * kVec;
    constexpr int U = kBulkRowsInFlight;
    constexpr int NG = B::kGroups;
    static_assert(32 % kLPR == 0 && B::kNV % kLPR == 0, "row must map onto a sub-warp");

    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kBulkStages * B::kChunkBytes);
    uint64_t *empty = full + kBulkStages;
    const int warp = threadIdx.x / 32;
    const uint64_t rows = (uint64_t)T * heads;
    const int64_t row_bytes_g = row_stride * (int64_t)sizeof(TS);  // token stride in bytes
    const bool contiguous = row_bytes_g == (int64_t)heads * B::kRowBytes;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kBulkStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kBulkConsumerWarps);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait_then_release();

    if (warp == 0) {
        // ---- producer: one lane issues the bulk copies of each chunk --
        if (threadIdx.x == 0) {
            const uint64_t policy = l2_evict_first_policy();
            const unsigned char *base = reinterpret_cast<const unsigned char *>(qkv);
            uint32_t k = 0;
            bool ok = true;
            for (uint64_t c = blockIdx.x; c < nchunks && ok; c += gridDim.x, ++k) {
                const uint32_t s = k % kBulkStages, n = k / kBulkStages;
                if (n > 0 && !mbar_wait_cta_bounded(&empty[s], (n - 1) & 1u)) {
                    atomicAdd(&g_wait_timeouts, 1u);
                    ok = false;
                    break;
                }
                const uint64_t r0 = c * B::kChunkRows;
                const uint64_t r1 = r0 + B::kChunkRows < rows ? r0 + B::kChunkRows : rows;
                unsigned char *dst = smem + (size_t)s * B::kChunkBytes;
                mbar_arm(&full[s], (uint32_t)((r1 - r0) * B::kRowBytes));
                if (contiguous) {
                    bulk_load(dst, base + r0 * B::kRowBytes, (uint32_t)((r1 - r0) * B::kRowBytes),
                              &full[s], policy);
                } else {
                    uint64_t t = r0 / heads;
                    uint32_t h = (uint32_t)(r0 - t * heads);
                    for (uint64_t r = r0; r < r1;) {
                        const uint64_t seg = (heads - h) < (r1 - r) ? (heads - h) : (r1 - r);
                        bulk_load(dst + (r - r0) * B::kRowBytes,
                                  base + (int64_t)t * row_bytes_g + (int64_t)h * B::kRowBytes,
                                  (uint32_t)(seg * B::kRowBytes), &full[s], policy);
                        r += seg;
                        h = 0;
                        ++t;
                    }
                }
            }
            // Leave no copy in flight: wait for the last stages issued.
            const uint32_t issued = k;
            for (uint32_t j = issued > kBulkStages ? issued - kBulkStages : 0; j < issued; ++j)
                if (!mbar_wait_cta_bounded(&full[j % kBulkStages], (j / kBulkStages) & 1u))
                    atomicAdd(&g_wait_timeouts, 1u);
        }
        return;
    }

    // ---- consumers --
    const uint32_t ct = threadIdx.x - 32;
    const uint32_t lane = ct % kLPR;
    const uint32_t g = ct / kLPR;  // row group, 0 .. NG-1
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
    // Row steps within a chunk, as (tokens, heads) with heads < `heads`: to
    // this thread's first row of slot u (u * NG + g), and from one pass to
    // the next (U * NG rows).
    uint32_t off_t[U], off_h[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const uint32_t r = (uint32_t)u * NG + g;
        off_t[u] = r / heads;
        off_h[u] = r - off_t[u] * heads;
    }
    const uint32_t step_t = (uint32_t)B::kPassRows / heads;
    const uint32_t step_h = (uint32_t)B::kPassRows - step_t * heads;
    unsigned char *gbase = reinterpret_cast<unsigned char *>(qkv);

    uint32_t k = 0;
    for (uint64_t c = blockIdx.x; c < nchunks; c += gridDim.x, ++k) {
        const uint32_t s = k % kBulkStages;
        // The whole warp goes on or stops together (its lanes shuffle).
        const bool ok = mbar_wait_cta_bounded(&full[s], (k / kBulkStages) & 1u);
        if (!__all_sync(0xffffffffu, ok)) {
            if ((threadIdx.x & 31) == 0) atomicAdd(&g_wait_timeouts, 1u);
            break;
        }
        const uint64_t r0 = c * B::kChunkRows;
        const uint64_t t0 = r0 / heads;
        const uint32_t h0 = (uint32_t)(r0 - t0 * heads);
        const uint32_t nrows = (uint32_t)(rows - r0 < (uint64_t)B::kChunkRows ? rows - r0
                                                                              : B::kChunkRows);
        const unsigned char *stage = smem + (size_t)s * B::kChunkBytes;
        int64_t t[U];
        uint32_t h[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            t[u] = (int64_t)t0 + off_t[u];
            h[u] = h0 + off_h[u];
            if (h[u] >= heads) {
                h[u] -= heads;
                t[u] += 1;
            }
        }
#pragma unroll 1
        for (uint32_t pr = 0; pr < (uint32_t)B::kChunkRows; pr += B::kPassRows) {
            V x[U][kVPL];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const uint32_t r = pr + (uint32_t)u * NG + g;
                const V *src = reinterpret_cast<const V *>(stage + (size_t)r * B::kRowBytes) + lane;
#pragma unroll
                for (int v = 0; v < kVPL; ++v) x[u][v] = r < nrows ? src[v * kLPR] : zero_vec<V>();
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                float f[kVPL][kVec];
                float sum = 0.f;
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    S::unpack(x[u][v], f[v]);
#pragma unroll
                    for (int e = 0; e < kVec; ++e) sum = fmaf(f[v][e], f[v][e], sum);
                }
                sum = group_sum<kLPR>(sum);
                const float rinv = rsqrtf(sum / (float)D + eps);
                const uint32_t r = pr + (uint32_t)u * NG + g;
                if (r < nrows) {
                    const bool is_q = !kHasK || h[u] < Hq;
                    V *dst = reinterpret_cast<V *>(gbase + t[u] * row_bytes_g +
                                                   (int64_t)h[u] * B::kRowBytes) +
                             lane;
#pragma unroll
                    for (int v = 0; v < kVPL; ++v) {
                        float o[kVec];
#pragma unroll
                        for (int e = 0; e < kVec; ++e) {
                            float gg = gq[v * kVec + e];
                            if constexpr (kHasK) gg = is_q ? gg : gk[v * kVec + e];
                            o[e] = f[v][e] * rinv * gg;
                        }
                        store_stream(dst + v * kLPR, S::pack(o));
                    }
                }
                t[u] += step_t;
                h[u] += step_h;
                if (h[u] >= heads) {
                    h[u] -= heads;
                    t[u] += 1;
                }
            }
        }
        // This warp has read the stage: one arrival per consumer warp frees it.
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(&empty[s]);
    }
}
