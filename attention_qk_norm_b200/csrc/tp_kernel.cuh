// tp_kernel.cuh -- tensor-parallel layerwise QK-Norm with the scalar exchange
// inside the kernel (qknorm_layerwise_tp_p2p).  The exchange protocol (slot
// layout, {value, tag} words, call parity, rank tree) is in tp_exchange.h.
// Part of libqknorm.so; included by qknorm.cu, the library's one translation
// unit.
//
// Each block takes tokens b, b + G, ... (G blocks per rank, the same on every
// rank) through a three-stage cp.async ring.  In iteration i it forms token
// t_i's head partials, meets the block at one barrier, and warp 0 stores the
// rank's two sums of t_i into every rank's receive buffer; then every warp
// finishes token t_{i-1}: it reads the world ranks' sums of t_{i-1} from
// this rank's buffer (sent one iteration earlier, so the exchange latency
// is hidden behind a token's load and partial sums), combines them with the
// fixed rank tree and scales the staged token.  The last token is finished
// after the loop.  This one-token lag is SwiftQK's overlap of the exchange
// with work (SwiftQK review, key_machinery), taken one token further than
// overlapping only the weight multiplication.
//
// Calls: the sequence number of the call (which picks the buffer half and
// the tag) is read from device memory when the launch starts and advanced by
// the launch's last block, so consecutive launches, replayed graphs
// included, always carry consecutive sequence numbers.
//
// Deadlock freedom: a block's poll for t_{i-1} waits for the blocks of the
// same index on the other ranks to have sent t_{i-1}, which each does in its
// iteration i-1 before it polls anything of iteration i-1 itself; so by
// induction over the iterations every poll is eventually satisfied, provided
// every block of every rank gets to run (no more blocks per rank than fit
// resident; a cooperative launch where one launch serves several ranks, whose
// blocks then wait on one another) and blocks take the same tokens on every
// rank.  Each poll still gives up after the
// communicator's time limit, and the first give-up stops every later wait of
// the call on this rank.
#pragma once

#include "layerwise.cuh"
#include "storage.cuh"
#include "tp_exchange.h"

namespace {

// The exchange of one launch.  The call's sequence number lives in device
// memory: every block reads it when the launch starts, and the last block to
// finish advances it, so launches replayed from a CUDA graph get new tags.
struct P2PArgs {
    uint64_t *recv[qkn_tp::kMaxWorld];  // every rank's receive buffer, as this GPU addresses it
    unsigned int *errors;               // the group's count of waits that gave up
    uint32_t *abort_tag;                // tag of a call in which a wait gave up
    uint32_t *seq;                      // calls made on this GPU's communicator so far
    uint32_t *done;                     // blocks of the current launch that have finished
    int64_t max_tokens;
    uint64_t timeout_ns;
    int world;
    int rank;                           // rank of grid row 0 (blockIdx.y adds to it)
};

// Pointers of the ranks one launch serves: one (a rank on its own GPU) or
// every rank of a group emulated on one GPU (grid row y serves rank
// p2p.rank + y).
struct TPRankPtrs {
    void *qkv[qkn_tp::kMaxWorld];
    const float *gamma_q[qkn_tp::kMaxWorld];
    const float *gamma_k[qkn_tp::kMaxWorld];
};

// 64-bit relaxed accesses at system scope: a peer's stores over NVLink and
// this GPU's polls of them.  Each is single-copy atomic (naturally aligned).
__device__ __forceinline__ void st_relaxed_sys_u64(uint64_t *p, uint64_t v)
{
    asm volatile("st.relaxed.sys.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ uint64_t ld_relaxed_sys_u64(const uint64_t *p)
{
    uint64_t v;
    asm volatile("ld.relaxed.sys.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu_u32(const uint32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Element i of a small pointer array held in kernel parameters, with a
// compile-time index on every access (no copy of the array to local memory).
template <typename P, int N>
__device__ __forceinline__ P pick(const P (&a)[N], int i)
{
    P r = a[0];
#pragma unroll
    for (int j = 1; j < N; ++j)
        if (j == i) r = a[j];
    return r;
}

constexpr int kTPStages = 3;

// Registers per thread of the exchange kernel: 48 with up to 16 elements per
// thread (no spills once the rank's sums use the warp tree; measured on B200
// it runs one rank's 32q/8kv tokens 4-17% faster than at 56, with a fourth
// resident 320-thread block per SM), 72 with 32.
__host__ __device__ constexpr int tp_regs(int ept) { return ept <= 16 ? 48 : 72; }

template <typename TS, int D, int VPT>
__global__ void __maxnreg__((tp_regs(VPT * Storage<TS>::kVec)))
qkn_layerwise_tp_kernel(TPRankPtrs ptrs, int64_t row_stride, int64_t T, int Hq, int Hk,
                        float eps, float inv_len_q, float inv_len_k, SumPlan plan_q,
                        SumPlan plan_k, P2PArgs p2p)
{
    using S = Storage<TS>;
    using V = typename S::Vec;
    constexpr int kVB = (int)sizeof(V);
    constexpr int kVec = S::kVec;
    constexpr int kNV = D / kVec;     // vectors per head
    constexpr int kLPH = kNV / VPT;   // threads per head
    constexpr int kEPT = VPT * kVec;  // elements per thread
    static_assert(kNV % VPT == 0 && 32 % kLPH == 0, "head must map onto a sub-warp");
    static_assert(kEPT <= 32, "gamma is held in registers");

    extern __shared__ __align__(16) unsigned char smem[];
    const int y = (int)blockIdx.y;
    const int me = p2p.rank + y;
    TS *qkv = static_cast<TS *>(pick(ptrs.qkv, y));
    const float *gamma_q = pick(ptrs.gamma_q, y), *gamma_k = pick(ptrs.gamma_k, y);
    const int heads = Hq + Hk;
    const int span = heads * D * (int)sizeof(TS);
    float *const part0 = reinterpret_cast<float *>(smem + (size_t)kTPStages * span);
    float *const part1 = part0 + heads;
    const int hl = threadIdx.x / kLPH;  // head
    const int l = threadIdx.x % kLPH;
    const bool active = hl < heads;
    const int lane = threadIdx.x % 32;
    const bool need_q = (int)((threadIdx.x & ~31) / kLPH) < Hq;
    const bool need_k = Hk > 0 && (int)((threadIdx.x | 31) / kLPH) >= Hq;
    const int world = p2p.world;
    const int64_t first = blockIdx.x, stride = gridDim.x;

    // This thread's vectors of its first token into L2 before the wait (a
    // hint that returns no data; see prefetch_l2).
    if (active && first < T) {
        const TS *row = qkv + first * row_stride + (int64_t)hl * D + l * kVec;
#pragma unroll
        for (int v = 0; v < VPT; ++v) prefetch_l2(row + v * kLPH * kVec);
    }
    pdl_wait_then_release();
    // This call's buffer half and tag (tp_exchange.h), from the sequence
    // number that the previous launch left behind.
    const uint32_t call = ld_relaxed_gpu_u32(p2p.seq);
    const uint32_t parity = qkn_tp::call_parity(call), tag = qkn_tp::call_tag(call);
    // Lane r of a warp stores to, and polls the slot of, rank r.
    uint64_t *const peer_buf = pick(p2p.recv, lane);
    const uint64_t *const own_buf = pick(p2p.recv, me);

    const float *gb = gamma_q;
    if (active) gb = hl < Hq ? gamma_q + (int64_t)hl * D : gamma_k + (int64_t)(hl - Hq) * D;
    float g[kEPT];
#pragma unroll
    for (int e = 0; e < kEPT; ++e) g[e] = 0.f;
    if (active) {
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            float t4[kVec];
            load_gamma<kVec>(gb + (l + v * kLPH) * kVec, t4);
#pragma unroll
            for (int e = 0; e < kVec; ++e) g[v * kVec + e] = t4[e];
        }
    }

    // Running addresses: this thread's first vector of its head in the row of
    // the current token, and its vectors in the three stages.
    const int64_t row_bytes = row_stride * (int64_t)sizeof(TS);
    const int64_t step_bytes = stride * row_bytes;
    const unsigned char *gcur = reinterpret_cast<const unsigned char *>(qkv) +
                                (int64_t)hl * D * (int64_t)sizeof(TS) + (int64_t)l * kVB +
                                first * row_bytes;
    const int scol0 = (hl * D + l * kVec) * (int)sizeof(TS);
    const V *sp_prev = reinterpret_cast<const V *>(smem + 2 * span + scol0);
    const V *sp_cur = reinterpret_cast<const V *>(smem + scol0);
    const V *sp_nxt = reinterpret_cast<const V *>(smem + span + scol0);
    auto fetch = [&](const unsigned char *src, int64_t tok, const V *dst) {
        if (active && tok < T) {
            const uint32_t d = smem_u32(dst);
#pragma unroll
            for (int v = 0; v < VPT; ++v)
                cp_async_s(d + (uint32_t)(v * kLPH * kVB), src + v * kLPH * kVB);
        }
        cp_async_commit();
    };

    bool gave_up = false;
    // Scale token t (staged at sp, row at grow) once the world ranks' sums of
    // t have arrived in this rank's buffer.
    auto finish = [&](int64_t t, const unsigned char *grow, const V *sp) {
        float rq = 0.f, rk = 0.f;
        if (need_q || need_k) {
            float vq = 0.f, vk = 0.f;
            bool ok = true;
            if (lane < world) {
                const uint64_t *src =
                    own_buf + qkn_tp::slot_word(parity, t, lane, 0, p2p.max_tokens, world);
                uint64_t wq = ld_relaxed_sys_u64(src), wk = ld_relaxed_sys_u64(src + 1);
                if (!gave_up && !(qkn_tp::arrived(wq, tag) && qkn_tp::arrived(wk, tag))) {
                    const uint64_t t0 = global_ns();
                    for (;;) {
                        wq = ld_relaxed_sys_u64(src);
                        wk = ld_relaxed_sys_u64(src + 1);
                        if (qkn_tp::arrived(wq, tag) && qkn_tp::arrived(wk, tag)) break;
                        if (global_ns() - t0 > p2p.timeout_ns ||
                            ld_relaxed_gpu_u32(p2p.abort_tag) == tag) {
                            ok = false;
                            break;
                        }
                    }
                }
                vq = qkn_tp::value_of(wq);
                vk = qkn_tp::value_of(wk);
            }
            if (__any_sync(0xffffffffu, !ok) && !gave_up) {
                // Count it, tell the other blocks, and wait no more in this
                // launch (its outputs are wrong from here on).
                gave_up = true;
                if (lane == 0) {
                    atomicAdd(p2p.errors, 1u);
                    atomicAdd(&g_wait_timeouts, 1u);
                    atomicExch(p2p.abort_tag, tag);
                }
            }
            for (int d = 1; d < world; d <<= 1) {  // the fixed rank tree (tp_exchange.h)
                vq += __shfl_xor_sync(0xffffffffu, vq, d);
                vk += __shfl_xor_sync(0xffffffffu, vk, d);
            }
            vq = __shfl_sync(0xffffffffu, vq, 0);
            vk = __shfl_sync(0xffffffffu, vk, 0);
            if (need_q) rq = rsqrtf(vq * inv_len_q + eps);
            if (need_k) rk = rsqrtf(vk * inv_len_k + eps);
        }
        if (active) {
            const float rinv = hl < Hq ? rq : rk;
            V *p = reinterpret_cast<V *>(const_cast<unsigned char *>(grow));
#pragma unroll
            for (int v = 0; v < VPT; ++v) {
                float f[kVec], o[kVec];
                S::unpack(sp[v * kLPH], f);
#pragma unroll
                for (int e = 0; e < kVec; ++e) o[e] = f[e] * g[v * kVec + e] * rinv;
                store_stream(p + v * kLPH, S::pack(o));
            }
        }
    };

    fetch(gcur, first, sp_cur);
    uint32_t it = 0;
    int64_t tprev = -1;
    const unsigned char *gprev = gcur;
    for (int64_t t = first; t < T; t += stride, ++it) {
        fetch(gcur + step_bytes, t + stride, sp_nxt);  // the stage of token t-2, finished
        cp_async_wait<1>();
        // This rank's partial of each of its heads for token t.
        uint64_t acc = f2_pack(0.f, 0.f);
#pragma unroll
        for (int v = 0; v < VPT; ++v) {
            float f[kVec];
            S::unpack(active ? sp_cur[v * kLPH] : zero_vec<V>(), f);
            sumsq_acc(acc, f);
        }
        const float s = group_sum<kLPH>(sumsq_total(acc));
        // Partials alternate between two buffers: the next write into this
        // one is for token t + 2 stride, after the next barrier, which warp 0
        // reaches only after reading it below.
        float *pp = (it & 1u) ? part1 : part0;
        const bool tree = (plan_q.warps | plan_k.warps) != 0;  // the warp tree (layerwise.cuh)
        if (tree) {
            float w = s;
#pragma unroll
            for (int o = kLPH; o < 32; o <<= 1) w += __shfl_xor_sync(0xffffffffu, w, o);
            if (lane == 0) pp[threadIdx.x / 32] = w;
        } else if (active && l == 0) {
            pp[hl] = s;
        }
        __syncthreads();
        if (threadIdx.x < 32) {  // warp 0 sends this rank's two sums to every rank
            float sq, sk;
            if (tree) {
                sq = plan_q.warps ? warp_tree_sum(pp, plan_q.warps) : 0.f;
                sk = plan_k.warps ? warp_tree_sum(pp + plan_q.warps, plan_k.warps) : 0.f;
            } else {
                sq = warp_sumsq(pp, plan_q, lane);
                sk = warp_sumsq(pp + Hq, plan_k, lane);
            }
            if (lane < world) {
                uint64_t *dst =
                    peer_buf + qkn_tp::slot_word(parity, t, me, 0, p2p.max_tokens, world);
                st_relaxed_sys_u64(dst, qkn_tp::pack(sq, tag));
                st_relaxed_sys_u64(dst + 1, qkn_tp::pack(sk, tag));
            }
        }
        if (tprev >= 0) finish(tprev, gprev, sp_prev);
        tprev = t;
        gprev = gcur;
        gcur += step_bytes;
        const V *tp = sp_prev;
        sp_prev = sp_cur;
        sp_cur = sp_nxt;
        sp_nxt = tp;
    }
    if (tprev >= 0) finish(tprev, gprev, sp_prev);
    cp_async_wait<0>();
    // The last block of the launch to finish advances the sequence number
    // (every block has read it by then: it read it before its first token).
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned int blocks = gridDim.x * gridDim.y;
        if (atomicAdd(p2p.done, 1u) == blocks - 1) {
            atomicExch(p2p.done, 0u);
            atomicAdd(p2p.seq, 1u);
        }
    }
}

}  // namespace
