// layerwise.cuh -- the layerwise QK-Norm kernel: the fixed reduction tree,
// the cluster exchange of head partials on transaction barriers, and the
// kernel entry points of its modes and variants.
// Part of libqknorm.so; included by qknorm.cu, the library's one translation
// unit.
#pragma once

#include <cooperative_groups.h>

#include "storage.cuh"

namespace {

// --------------------------------------------------------------- layerwise --

// How warp_sumsq reduces the nh head partials of one vector (q or k).  The
// host fills it once per launch, so the token loop divides nothing.
//   used:      lanes that hold partials, min(p, 32) with p the largest power
//              of two dividing nh (0 when nh == 0);
//   per_lane:  heads each of those lanes sums, in order (nh / used);
//   per_shard: lanes per emulated shard (used / nshards).
//   warps:     with the warp tree (below), the warps whose sums make up
//              the vector (0 for both vectors when it is not used).
struct SumPlan {
    int used;
    int per_lane;
    int per_shard;
    int warps;
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
//
// The butterflies at distances below per_shard and those above it are one
// sequence of xor steps (distance 1, 2, 4, ... below `used`), unrolled here
// with each step predicated on the warp-uniform plan.
__device__ __forceinline__ float warp_sumsq(const float *part, const SumPlan &p, int lane)
{
    float v = 0.f;
    if (lane < p.used) {  // used > 0 means per_lane >= 1
        const float *q = part + lane * p.per_lane;
        v = q[0];
        for (int j = 1; j < p.per_lane; ++j) v += q[j];
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1)
        if (o < p.used) v += __shfl_xor_sync(0xffffffffu, v, o);
    return __shfl_sync(0xffffffffu, v, 0);
}

// The warp tree.  When a vector's head count nh is a power of two up to 64,
// warp_sumsq's tree is the balanced binary tree over head index (with 64
// heads each lane first adds two neighbours, which is the tree's lowest
// level).  A block of a plain launch with gamma in registers, whose warps
// each hold hpw = 32 / LPH whole heads of one vector (hpw dividing Hq),
// then holds that tree's subtrees warp by warp: each warp forms its subtree
// with xor butterflies at lane distances LPH, 2 LPH, ... 16 (head distances
// 1, 2, ..., hpw / 2) before the block barrier, and after it every lane adds
// the vector's n <= 8 warp sums in the tree's remaining levels.  The
// association is the same, so the bits are too; lanes past the last head add
// zeros, which leaves a sum of squares unchanged.
__device__ __forceinline__ float warp_tree_sum(const float *w, int n)
{
    if (n == 1) return w[0];
    if (n == 2) return w[0] + w[1];
    if (n == 4) return (w[0] + w[1]) + (w[2] + w[3]);
    return ((w[0] + w[1]) + (w[2] + w[3])) + ((w[4] + w[5]) + (w[6] + w[7]));
}

// ---- cluster exchange of head partials (transaction barriers) --
// Each block of a cluster keeps two mbarriers, one per partials buffer.  The
// owner of a head pushes that head's fp32 partial into the buffer of every
// block of the cluster with st.async, which also counts its 4 bytes against
// the receiving block's barrier; a block's barrier phase completes once all
// (Hq + Hk) partials of the token have landed and its own thread 0 has armed
// the phase.  No cluster-wide barrier and no memory fence is on the token path.
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

// How a launch moves each token through its block.
//   kSchedRing:    a cp.async ring in shared memory (the next token is
//                  fetched while this one is processed; layerwise_stages),
//                  then a second pass over the staged token to scale it.
//   kSchedOverlap: the ring, with x * gamma formed in the first pass, while
//                  the token's partials are still being combined (SwiftQK's
//                  overlap), and kept in registers: no second pass.
//   kSchedDirect:  for launches where every cluster has about one token, so
//                  there is nothing to prefetch: each thread loads its vectors
//                  straight into registers and scales them there; nothing is
//                  staged.
enum LayerwiseSchedule { kSchedRing = 0, kSchedOverlap = 1, kSchedDirect = 2 };

// Stages of the staging ring: two (one token staged ahead of the one being
// worked on), three for FP8 on the overlap schedule.  Measured on B200: a
// third stage costs bf16/fp16/fp32 2-11% (a resident block fewer, or, for
// fp32 on the overlap schedule, 2-9% with the same blocks), while FP8, whose
// tokens are short and whose four resident blocks keep only 20 KB per SM in
// flight with two stages, gains 4-5% (32q/8kv, T = 8192 to 32768); a fourth
// stage is slower again.
template <typename TS, int kSched>
__host__ __device__ constexpr int layerwise_stages()
{
    return kSched == kSchedDirect                                  ? 0
           : (kSched == kSchedOverlap && Storage<TS>::kVec == 16) ? 3
                                                                  : 2;
}

// A token's heads are split over the CL blocks of a thread-block cluster
// (CL = 1 for a plain launch): block c of a cluster owns heads
// [c*hc, (c+1)*hc), hc = heads/CL, with roundup32(hc * NV / VPT) threads;
// thread (h, l) owns vectors l, l + LPH, ... of head h (LPH = NV / VPT lanes
// per head), and thread l == 0 is the head's owner.  Dynamic shared memory
// per block: the ring's layerwise_stages() stages of this block's part of a
// token (hc*D*sizeof(TS) bytes each; none with the direct schedule), two
// buffers of `heads` fp32 head partials (alternating per token), then the
// two exchange barriers (CL > 1).  With
// CL = 1 the partials meet behind one block barrier per token; with CL > 1
// each owner pushes its partial into every block of the cluster and each
// block waits on its own barrier (see the exchange helpers above).
template <typename TS, int D, int VPT, bool kGammaRegs, bool kCluster, int kMode, int kSched>
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
    constexpr bool kOverlap = kSched == kSchedOverlap;
    constexpr bool kDirect = kSched == kSchedDirect;
    // Every schedule sums squares in f32x2 pairs (sumsq_acc), so a head's
    // partial is the same bits in every mode and schedule; the overlap
    // schedule also forms its products on pairs, while the others, whose
    // register caps leave no room for pair alignment, multiply in scalars
    // (the same bits either way).
    constexpr bool kPacked = kOverlap;
    constexpr int NST = layerwise_stages<TS, kSched>();  // stages of the ring
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

    // This thread's vectors of the first tokens (those the ring stages first,
    // or the one the direct schedule loads) into L2 before the wait.  Not in
    // the apply step, which follows the all-reduce (a grid that lets no
    // dependent start early), nor with gamma read through L1.
    if constexpr (kGammaRegs && kMode != kApply) {
        if (active) {
            const TS *row = qkv + first * row_stride + (int64_t)h * D + l * kVec;
#pragma unroll
            for (int i = 0; i < (NST > 1 ? NST - 1 : 1); ++i)
                if (first + i * stride < T) {
#pragma unroll
                    for (int v = 0; v < VPT; ++v)
                        prefetch_l2(row + i * stride * row_stride + v * kLPH * kVec);
                }
        }
    }
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
    static_assert(kDirect || NST >= 2, "the ring has at least two stages");
    // Running addresses, advanced per token instead of recomputed: this
    // thread's first vector of head h in the row of its current token (the
    // row advances by step_bytes), and its vectors in the ring's stages.
    // Each thread copies, and later reads, only its own vectors of a stage.
    const int64_t row_bytes = row_stride * (int64_t)sizeof(TS);
    const int64_t step_bytes = stride * row_bytes;
    const unsigned char *gcur = reinterpret_cast<const unsigned char *>(qkv) +
                                (int64_t)h * D * (int64_t)sizeof(TS) + (int64_t)l * kVB +
                                first * row_bytes;
    const int scol0 = (hl * D + l * kVec) * (int)sizeof(TS);  // in a stage
    // Byte offsets of the stage being worked on and of the stage being
    // refilled (NST - 1 tokens ahead), each wrapping at the ring's end.
    const uint32_t ring = (uint32_t)(NST > 0 ? NST : 1) * (uint32_t)span;
    const unsigned char *sbase = smem + scol0;
    const uint32_t ss_base = smem_u32(sbase);
    uint32_t off_cur = 0, off_fill = (uint32_t)(NST > 0 ? NST - 1 : 0) * (uint32_t)span;
    float *const part0 = part, *const part1 = part + heads;
    auto fetch = [&](const unsigned char *src, int64_t tok, uint32_t dst) {
        if (active && tok < T) {
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v)
                cp_async_s(dst + (uint32_t)(v * kLPH * kVB), src + v * kLPH * kVB);
        }
        cp_async_commit();
    };
    const unsigned char *gfill = gcur;  // row of the next token to stage
    int64_t tfill = first;
    if constexpr (!kDirect) {
#pragma unroll
        for (int i = 0; i < NST - 1; ++i) {
            fetch(gfill, tfill, ss_base + (uint32_t)(i * span));
            gfill += step_bytes;
            tfill += stride;
        }
    }
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
    uint32_t it = 0;  // tokens this block has done; partials buffer it % 2
    bool timed_out = false;
    for (int64_t t = first; t < T; t += stride, ++it) {
        // this thread's vectors of the token, staged (ring)
        const V *sp = reinterpret_cast<const V *>(sbase + off_cur);
        V xr[kDirect ? VPT : 1];  // or in registers (direct)
        if constexpr (kDirect) {
            const V *src = reinterpret_cast<const V *>(gcur);
#pragma unroll
            for (int v = 0; v < VPT; ++v)
                xr[v] = active ? load_stream(src + v * kLPH) : zero_vec<V>();
        } else {
            // Refill the stage this thread finished with on the previous token.
            fetch(gfill, tfill, ss_base + off_fill);
            gfill += step_bytes;
            tfill += stride;
            cp_async_wait<(NST > 0 ? NST - 1 : 0)>();
        }
        float rq = 0.f, rk = 0.f;
        float xg[kOverlap ? kEPT : 1];  // x * gamma, formed before the combine
        if constexpr (kMode == kApply) {
            // Sums over all ranks come in; no exchange inside the launch.
            if (Hq > 0) rq = rsqrtf(__ldg(aux + 2 * t) * inv_len_q + eps);
            if (Hk > 0) rk = rsqrtf(__ldg(aux + 2 * t + 1) * inv_len_k + eps);
        } else {
            float s = 0.f;
            uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v) {
                float f[kVec];
                if constexpr (kDirect)
                    S::unpack(xr[v], f);
                else
                    S::unpack(active ? sp[v * kLPH] : zero_vec<V>(), f);
                sumsq_acc(acc, f);
                if constexpr (kPacked) {
                    float t[kVec];
                    mul_elems(t, f, g + v * kVec);
#pragma unroll
                    for (int e = 0; e < kVec; ++e) xg[v * kVec + e] = t[e];
                } else if constexpr (kOverlap) {
#pragma unroll
                    for (int e = 0; e < kVec; ++e) xg[v * kVec + e] = f[e] * g[v * kVec + e];
                }
            }
            s = sumsq_total(acc);
            s = group_sum<kLPH>(s);
            // Partials alternate between two buffers.  The next write into
            // this token's buffer is for the token after next; every block
            // sends it only after the token in between, which needs a partial
            // from every warp of the cluster, and each warp sends that only
            // after it has finished reading this buffer.  (Every warp holds an
            // owner: its first thread.)
            const uint32_t pb = it & 1u;
            float *pp = pb ? part1 : part0;
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
            } else if (kGammaRegs && (plan_q.warps | plan_k.warps)) {
#pragma unroll
                for (int o = kLPH; o < 32; o <<= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
                if (lane == 0) pp[threadIdx.x / 32] = s;
                __syncthreads();
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
            } else if (kGammaRegs && !kExchange && (plan_q.warps | plan_k.warps)) {
                if (need_q) rq = rsqrtf(warp_tree_sum(pp, plan_q.warps) * inv_len_q + eps);
                if (need_k)
                    rk = rsqrtf(warp_tree_sum(pp + plan_q.warps, plan_k.warps) * inv_len_k + eps);
            } else {
                if (need_q) rq = rsqrtf(warp_sumsq(pp, plan_q, lane) * inv_len_q + eps);
                if (need_k) rk = rsqrtf(warp_sumsq(pp + Hq, plan_k, lane) * inv_len_k + eps);
            }
        }
        if (kMode != kPartials && active) {
            const float rinv = h < Hq ? rq : rk;
            V *p = reinterpret_cast<V *>(const_cast<unsigned char *>(gcur));
#pragma unroll kUnroll
            for (int v = 0; v < VPT; ++v) {
                float o[kVec];
                if constexpr (kPacked) {
                    mul_scalar(o, xg + v * kVec, rinv);
                } else if constexpr (kOverlap) {
#pragma unroll
                    for (int e = 0; e < kVec; ++e) o[e] = xg[v * kVec + e] * rinv;
                } else {
                    float f[kVec], gv[kVec];
                    if constexpr (kDirect)
                        S::unpack(xr[v], f);
                    else
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
                store_stream(p + v * kLPH, S::pack(o));
            }
        }
        gcur += step_bytes;
        if constexpr (!kDirect) {
            off_fill = off_cur;
            off_cur += (uint32_t)span;
            if (off_cur == ring) off_cur = 0;
        }
    }
    cp_async_wait<0>();
    // No block leaves while a partner could still write into it.
    if constexpr (kExchange) cooperative_groups::this_cluster().sync();
}

// Registers per thread: 40, 48 or 56 when a thread keeps 8, 16 or 32
// elements (and as many gamma values) per token.  The caps fit without
// spilling and leave room for more resident blocks than the compiler's own
// choice (up to 64); measured on B200 they are the fastest for every storage
// type and head_dim.  FP8 threads with 32 elements (two 16-element vectors)
// need 64 to decode a vector without spilling.  The overlap and direct
// schedules also keep the thread's x * gamma products, or its raw vectors,
// in registers: 48, 64 or 96.
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
#ifndef QKN_LW_REGS32_FP8
#define QKN_LW_REGS32_FP8 64
#endif
__host__ __device__ constexpr int layerwise_regs(int ept, bool wide, int kvec)
{
    return wide ? (ept <= 8 ? QKN_LW_OVERLAP_REGS8
                               : (ept <= 16 ? QKN_LW_OVERLAP_REGS16 : QKN_LW_OVERLAP_REGS32))
                   : (ept <= 8 ? QKN_LW_REGS8
                               : (ept <= 16 ? QKN_LW_REGS16
                                            : (kvec == 16 ? QKN_LW_REGS32_FP8 : QKN_LW_REGS32)));
}

// Gamma in registers (at most 32 elements per thread), with schedule kSched
// (LayerwiseSchedule).  With kSchedOverlap each thread forms x * gamma while
// the token's partials are still being combined (SwiftQK's overlap of the
// weight multiplication with the exchange), so after the combine only the
// multiplication by the inverse RMS remains.
template <typename TS, int D, int VPT, bool kCluster, int kMode, int kSched>
__global__ void __maxnreg__((layerwise_regs(VPT * Storage<TS>::kVec, kSched != kSchedRing,
                                             Storage<TS>::kVec)))
qkn_layerwise_kernel(TS *__restrict__ qkv, int64_t row_stride, int64_t T, int Hq, int Hk,
                     const float *__restrict__ gamma_q, const float *__restrict__ gamma_k,
                     float eps, float inv_len_q, float inv_len_k, SumPlan plan_q,
                     SumPlan plan_k, float *__restrict__ aux)
{
    layerwise_tokens<TS, D, VPT, true, kCluster, kMode, kSched>(
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
    layerwise_tokens<TS, D, VPT, false, false, kMode, kSchedRing>(
        qkv, row_stride, T, Hq, Hk, gamma_q, gamma_k, eps, inv_len_q, inv_len_k, plan_q, plan_k,
        aux);
}

}  // namespace
