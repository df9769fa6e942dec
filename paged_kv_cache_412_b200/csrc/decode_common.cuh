// decode_common.cuh -- work decomposition shared by the decode kernels.
//
// The work of one decode call is the flattened list of CH-token chunks over
// (request b, head group hg, chunk c), in that order; a head group is one kv
// head with the query heads that read it.  The list is cut into units of W
// consecutive chunks and CTA x processes units x, x + gridDim.x, ...  Inside a
// unit the chunks form segments, maximal runs inside one (b, hg).  Producer
// and consumer warps walk the same segments in the same order.

#pragma once

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {

__device__ __forceinline__ int clamp_len(const DecodeParams& p, int b, bool flag) {
    int L = __ldg(p.seq_lens + b);
    const int cap = p.max_blocks * p.block_size;
    if (L < 0 || L > cap) {
        if (flag) raise_error(p.err, PKV_DEVERR_BAD_SEQ_LEN);
        L = L < 0 ? 0 : cap;
    }
    return L;
}

template <int CH>
__device__ __forceinline__ int chunks_of(int L) {
    return (L + CH - 1) / CH;
}


// ---- shared prefixes --------------------------------------------------------
// A prefix group is a set of requests whose block tables name the same
// physical blocks for their first prefix_lens[g] tokens (blocks a fork shares).
// The shared pass reads those tokens once for the whole group and leaves
// per-(request, query head) partial results; the per-request pass then starts
// at the prefix's end and folds them in.

constexpr int kPrefixCH = 64;  // tokens per chunk of the shared pass

// Tokens the shared pass of group `g` covers: prefix_lens[g] clamped to
// [0, min(max_prefix_len, cap)] and rounded down to whole blocks, so both
// passes split every request at the same block boundary.  A length that needs
// clamping or rounding raises PKV_DEVERR_PREFIX when `flag`.
__device__ __forceinline__ int prefix_tokens(const int32_t* prefix_lens, int g, int max_prefix_len,
                                             int cap, int log2_bs, unsigned* err, bool flag) {
    const int raw = __ldg(prefix_lens + g);
    int t = min(max(raw, 0), min(max_prefix_len, cap));
    t = (t >> log2_bs) << log2_bs;
    if (flag && t != raw) raise_error(err, PKV_DEVERR_PREFIX);
    return t;
}

// The shared pass cuts a prefix of `ptok` tokens into splits of W chunks,
// W = ceil(chunks / S) for the S splits the launch provides; returns the
// number of splits that hold chunks (records the per-request pass folds in).
__device__ __forceinline__ int prefix_chunk_span(int ptok, int S) {
    const int nch = (ptok + kPrefixCH - 1) / kPrefixCH;
    return nch == 0 ? 0 : (nch + S - 1) / S;
}
__device__ __forceinline__ int prefix_num_splits(int ptok, int S) {
    const int nch = (ptok + kPrefixCH - 1) / kPrefixCH;
    if (nch == 0) return 0;
    const int w = (nch + S - 1) / S;
    return (nch + w - 1) / w;
}

// First token of request b's own pass (0 without a prefix group): the
// group's shared tokens, or all L of them if the request is shorter.
__device__ __forceinline__ int seq_begin(const DecodeParams& p, int b, int L, bool flag = false) {
    if (!p.prefix_of) return 0;
    const int g = __ldg(p.prefix_of + b);
    if (g < 0) return 0;
    if (g >= p.num_prefixes) {
        if (flag) raise_error(p.err, PKV_DEVERR_PREFIX);
        return 0;
    }
    const int t = prefix_tokens(p.prefix_lens, g, p.max_prefix_len, p.max_blocks * p.block_size,
                                p.log2_bs, p.err, flag);
    return min(t, L);
}

// Position in the flattened (request, head group, chunk) list.
struct Cursor {
    int b, hg, c, nch, L;
    int t0;  // first token of the request's pass (its chunk c starts at t0 + c*CH)
};

// Warp-cooperative search for global chunk index s (all lanes get the result).
// L_first, if >= 0, is this lane's (clamped) length of request `lane`, already
// loaded by the caller; it saves a dependent global load on the first pass.
template <int CH>
__device__ Cursor locate(const DecodeParams& p, long long s, int lane, int L_first = -1,
                         int T_first = 0) {
    Cursor cur{p.num_seqs, 0, 0, 0, 0, 0};
    long long base = 0;
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        int L = 0, T = 0;
        if (b < p.num_seqs) {
            if (b0 == 0 && L_first >= 0) {
                L = L_first;
                T = T_first;
            } else {
                L = clamp_len(p, b, false);
                T = seq_begin(p, b, L);
            }
        }
        const long long n = (long long)chunks_of<CH>(L - T) * p.num_hg;
        long long incl = n;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long t = __shfl_up_sync(FULL_MASK, incl, off);
            if (lane >= off) incl += t;
        }
        const long long excl = incl - n;
        const unsigned hit = __ballot_sync(FULL_MASK, n > 0 && base + excl <= s && s < base + incl);
        if (hit) {
            const int src = __ffs(hit) - 1;
            const int Lb = __shfl_sync(FULL_MASK, L, src);
            const int Tb = __shfl_sync(FULL_MASK, T, src);
            const long long ex = __shfl_sync(FULL_MASK, excl, src);
            const long long off = s - (base + ex);
            const int nch = chunks_of<CH>(Lb - Tb);
            cur.b = b0 + src;
            cur.L = Lb;
            cur.t0 = Tb;
            cur.nch = nch;
            cur.hg = (int)(off / nch);
            cur.c = (int)(off % nch);
            return cur;
        }
        base += __shfl_sync(FULL_MASK, incl, 31);
    }
    return cur;
}

// Move to chunk 0 of the next non-empty (request, head group).
template <int CH>
__device__ __forceinline__ void next_group(const DecodeParams& p, Cursor& cur) {
    cur.c = 0;
    if (++cur.hg < p.num_hg) return;
    cur.hg = 0;
    for (;;) {
        if (++cur.b >= p.num_seqs) {
            cur.nch = 0;
            return;
        }
        cur.L = clamp_len(p, cur.b, false);
        cur.t0 = seq_begin(p, cur.b, cur.L);
        cur.nch = chunks_of<CH>(cur.L - cur.t0);
        if (cur.nch > 0) return;
    }
}

// Total chunk count of the call, computed by the whole CTA (same in every CTA).
// `red` needs one long long per warp.
template <int CH>
__device__ long long total_chunks(const DecodeParams& p, long long* red, bool flag) {
    long long local = 0;
    for (int b = threadIdx.x; b < p.num_seqs; b += blockDim.x) {
        const int L = clamp_len(p, b, flag);
        local += chunks_of<CH>(L - seq_begin(p, b, L, flag));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(FULL_MASK, local, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
    __syncthreads();
    long long total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += red[w];
    return total * p.num_hg;
}

// One segment: chunks [c0, c1) of (cur.b, cur.hg) inside unit u.
struct Segment {
    Cursor cur;
    int c0, c1;
    long long u;        // unit
    long long gstart;   // global index of chunk 0 of (b, hg)
};

// Iterates this CTA's segments across all of its units.
template <int CH>
struct SegIter {
    long long total, W, nunits;
    long long u, s1, g;
    Cursor cur;
    bool valid;
    int L_first = -1;  // this lane's length of request `lane` (first 32 requests)
    int T_first = 0;   // and the first token of its pass

    __device__ void start_unit(const DecodeParams& p, int lane) {
        valid = u < nunits;
        if (!valid) return;
        const long long s0 = u * W;
        s1 = min(s0 + W, total);
        g = s0;
        cur = locate<CH>(p, s0, lane, L_first, T_first);
        valid = cur.nch > 0;
    }

    __device__ void init(const DecodeParams& p, long long total_, long long W_, int lane,
                         int L_first_ = -1, int T_first_ = 0) {
        total = total_;
        W = W_;
        nunits = (total + W - 1) / W;
        u = blockIdx.x;
        L_first = L_first_;
        T_first = T_first_;
        start_unit(p, lane);
    }

    __device__ __forceinline__ Segment current() const {
        Segment s;
        s.cur = cur;
        s.c0 = cur.c;
        s.c1 = (int)min((long long)cur.nch, (long long)cur.c + (s1 - g));
        s.u = u;
        s.gstart = g - cur.c;
        return s;
    }

    __device__ void advance(const DecodeParams& p, int lane) {
        const Segment s = current();
        g += s.c1 - s.c0;
        if (g < s1) {
            next_group<CH>(p, cur);
            valid = cur.nch > 0;
        } else {
            u += gridDim.x;
            start_unit(p, lane);
        }
    }
};

// Pipeline position in a ring of NSTAGE stages.
struct Ring {
    int stage = 0;
    uint32_t phase = 0;
    __device__ __forceinline__ void advance(int nstage) {
        if (++stage == nstage) {
            stage = 0;
            phase ^= 1u;
        }
    }
};

}  // namespace pkv
