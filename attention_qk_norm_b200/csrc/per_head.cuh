// per_head.cuh -- the per-head QK-Norm kernel.
// Part of libqknorm.so; included by qknorm.cu, the library's one translation
// unit.
#pragma once

#include "storage.cuh"

namespace {

// ---------------------------------------------------------------- per-head --
constexpr int kPerHeadThreads = 256;
constexpr int kPerHeadRowsInFlight = 2;
// Rows a thread keeps in flight per iteration, by storage type.  FP8 rows
// carry half the bytes of 16-bit ones, and with their sums and products on
// f32x2 pairs three fit the four-blocks-per-SM budget (64 registers, no
// spills): measured on B200, 0.81 -> 0.88 of the copy bandwidth on the GQA
// layout at T = 16384 and 0.86 -> 0.93-0.95 on wider shapes.  Three 16-bit
// or fp32 rows cost resident blocks and measured 2-6% slower.
template <typename TS>
constexpr int per_head_rows_in_flight()
{
    return Storage<TS>::kVec == 16 ? 3 : kPerHeadRowsInFlight;
}
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
    // FP8 rows (16 elements per lane) do their sums of squares (even and odd
    // elements in the two lanes of a pair) and products on f32x2 pairs, which
    // measured 2.5% faster on B200; the other types measured 0.5-1% faster in
    // scalars.
    constexpr bool kPacked = kVec == 16;

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

    // The first rows' (token, head) pairs depend on the arguments only: they
    // are found, and the rows' lines prefetched into L2, before the wait.
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
    // Rows of the first iteration, and of the second too when the launch has
    // at most four iterations: measured on B200, prefetching two iterations
    // gains 2-18% on such launches (48 heads at T = 1024 and 2048, 16 heads
    // at T = 4096) and costs 1-3% on longer ones.  Not with three rows in
    // flight, whose register budget it exceeds.
    const uint64_t rows = (uint64_t)T * heads;
    const int pf_iters = U == 2 && rows <= 4 * step ? 2 : 1;
#pragma unroll
    for (int k = 0; k < U; ++k) {
        int64_t tp = t[k];
        uint32_t hp = h[k];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            if (j < pf_iters && tp < T) {
                const V *p = reinterpret_cast<const V *>(qkv + tp * row_stride + (int64_t)hp * D);
#pragma unroll
                for (int v = 0; v < kVPL; ++v) prefetch_l2(p + lane + v * kLPR);
            }
            hp += dh;
            tp += dt;
            if (hp >= heads) {
                hp -= heads;
                tp += 1;
            }
        }
    }
    pdl_wait_then_release();

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
            if constexpr (kPacked) {
                uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    S::unpack(x[k][v], f[v]);
                    sumsq_acc(acc, f[v]);
                }
                s = sumsq_total(acc);
            } else {
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    S::unpack(x[k][v], f[v]);
#pragma unroll
                    for (int e = 0; e < kVec; ++e) s = fmaf(f[v][e], f[v][e], s);
                }
            }
            s = group_sum<kLPR>(s);
            const float rinv = rsqrtf(s / (float)D + eps);
            if (t[k] < T) {
                const bool is_q = !kHasK || h[k] < Hq;
#pragma unroll
                for (int v = 0; v < kVPL; ++v) {
                    float o[kVec];
                    if constexpr (kPacked) {
                        float g[kVec];
#pragma unroll
                        for (int e = 0; e < kVec; ++e) {
                            g[e] = gq[v * kVec + e];
                            if constexpr (kHasK) g[e] = is_q ? g[e] : gk[v * kVec + e];
                        }
                        mul_scalar(o, f[v], rinv);
                        mul_elems(o, o, g);
                    } else {
#pragma unroll
                        for (int e = 0; e < kVec; ++e) {
                            float g = gq[v * kVec + e];
                            if constexpr (kHasK) g = is_q ? g : gk[v * kVec + e];
                            o[e] = f[v][e] * rinv * g;
                        }
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
