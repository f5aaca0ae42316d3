// tp_exchange.h -- the scalar exchange of tensor-parallel layerwise QK-Norm
// done inside the kernel, as SwiftQK does it (SwiftQK abstract: ranks
// exchange only scalar statistics; SwiftQK review, key_machinery: warp 0
// writes its partial sums to the peers' buffers and waits on flags, then
// every element is scaled by 1/sqrt(S_global/H + eps)).
//
// Each rank owns a receive buffer in its own device memory, which the other
// ranks of the group write through CUDA IPC mappings (plain point-to-point
// peer stores over NVLink, one destination each).  For every token a rank stores its two fp32 partial
// sums of squares (its q heads, its k heads) into its slot of every rank's
// buffer, itself included, each as ONE 64-bit word {fp32 value, 32-bit call
// tag}: value and flag travel in a single naturally aligned store, so a
// reader that sees the tag of the current call sees that call's value, with
// no fence between a payload and a separate flag (the ordering question the
// review raises, major_comments[2]).  A reader polls the world slots of a
// token in its own buffer until all carry the current tag, with a time limit.
//
// Calls alternate between two halves of the buffer (the parity of the call
// counter), and a call's tag is never seen in a slot before that call writes
// it (tags grow by one per call of the same parity and start at 1 on a
// zeroed buffer).  A rank can run at most one call ahead of the slowest
// rank: it finishes call c only after every rank has sent its call-c sums
// for every token, which each rank does only after its call c-1 has ended,
// so the half that call c+1 writes is never still being read for call c-1.
//
// The rank sums are combined in a fixed pairwise tree in rank order (an xor
// butterfly at distances 1, 2, 4), so every rank gets the same bits.
//
// This header is shared by the CUDA kernel and a host build of the same
// protocol that the CPU tests drive with one process per rank; it holds
// only index arithmetic and the word format.
#pragma once

#include <stdint.h>
#include <string.h>

#if defined(__CUDACC__)
#define QKN_TP_HD __host__ __device__ __forceinline__
#else
#define QKN_TP_HD inline
#endif

namespace qkn_tp {

constexpr int kMaxWorld = 8;
constexpr int kWordsPerSlot = 2;  // the q sum and the k sum of one rank for one token

// Words in one rank's receive buffer: [2 halves][max_tokens][world][2].
QKN_TP_HD uint64_t buffer_words(int64_t max_tokens, int world)
{
    return 2ull * (uint64_t)max_tokens * (uint64_t)world * kWordsPerSlot;
}

// Index of word `which` (0: q, 1: k) of rank `src`'s slot for token t in the
// half of parity `parity`.
QKN_TP_HD uint64_t slot_word(uint32_t parity, int64_t t, int src, int which, int64_t max_tokens,
                             int world)
{
    return (((uint64_t)(parity & 1u) * (uint64_t)max_tokens + (uint64_t)t) * (uint64_t)world +
            (uint64_t)src) *
               kWordsPerSlot +
           (uint64_t)which;
}

// Parity and tag of the call with (0-based) sequence number `call`, a 32-bit
// count of the communicator's calls: the parity alternates, the tag grows by
// one per call of the same parity and is never 0 (the value of a slot never
// written).  After 2^32 calls the count wraps and tags repeat; a slot could
// then be taken for fresh only if no call in those 2^32 wrote it.
QKN_TP_HD uint32_t call_parity(uint32_t call) { return call & 1u; }
QKN_TP_HD uint32_t call_tag(uint32_t call) { return (call >> 1) + 1u; }

QKN_TP_HD uint32_t f32_bits(float v)
{
#if defined(__CUDA_ARCH__)
    return __float_as_uint(v);
#else
    uint32_t u;
    memcpy(&u, &v, 4);
    return u;
#endif
}
QKN_TP_HD float f32_from_bits(uint32_t u)
{
#if defined(__CUDA_ARCH__)
    return __uint_as_float(u);
#else
    float v;
    memcpy(&v, &u, 4);
    return v;
#endif
}

QKN_TP_HD uint64_t pack(float value, uint32_t tag) { return ((uint64_t)tag << 32) | f32_bits(value); }
QKN_TP_HD bool arrived(uint64_t word, uint32_t tag) { return (uint32_t)(word >> 32) == tag; }
QKN_TP_HD float value_of(uint64_t word) { return f32_from_bits((uint32_t)word); }

// The rank combine as lane 0 of an xor butterfly computes it (lane r holds
// s[r]; lanes at and beyond `world` hold 0): at distance d every lane adds
// its partner's value, d = 1, 2, 4 while d < world.  Host form, for the
// tests; the kernel runs the butterfly with shuffles.
inline float combine_ranks_host(const float *s, int world)
{
    float v[kMaxWorld];
    for (int r = 0; r < kMaxWorld; ++r) v[r] = r < world ? s[r] : 0.f;
    for (int d = 1; d < world; d <<= 1) {
        float n[kMaxWorld];
        for (int r = 0; r < kMaxWorld; ++r) n[r] = v[r] + v[r ^ d];
        for (int r = 0; r < kMaxWorld; ++r) v[r] = n[r];
    }
    return v[0];
}

}  // namespace qkn_tp
