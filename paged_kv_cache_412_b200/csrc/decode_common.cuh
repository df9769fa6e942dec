// decode_common.cuh -- work decomposition shared by the decode kernels.
//
// The work of one decode call is the flattened list of CH-token chunks over
// (request b, head group hg, chunk c), in that order; a head group is one kv
// head with the query heads that read it.  The list is cut into units of W
// consecutive chunks and CTA x processes units x, x + gridDim.x, ...  Inside a
// unit the chunks form segments, maximal runs inside one (b, hg).  Producer
// and consumer warps walk the same segments in the same order.
//
// With dynamic tails on (tail_chunks > 0) the list holds all but the last
// tail_chunks chunks of every (b, hg); those tails are handed out one (b, hg)
// at a time, by an atomic ticket, to whichever CTAs finish their static unit
// first, so CTAs on faster SMs take more of the work.
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

// Chunks of a (request, head group) pass of n tokens in the static list: all
// of them, or all but the last tail_chunks when the dynamic tails are on.
template <int CH>
__device__ __forceinline__ int list_chunks(const DecodeParams& p, int n) {
    return max(chunks_of<CH>(n) - p.tail_chunks, 0);
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
        const long long n = (long long)list_chunks<CH>(p, L - T) * p.num_hg;
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
            const int nch = list_chunks<CH>(p, Lb - Tb);
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
        cur.nch = list_chunks<CH>(p, cur.L - cur.t0);
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
        local += list_chunks<CH>(p, L - seq_begin(p, b, L, flag));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(FULL_MASK, local, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
    __syncthreads();
    long long total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) total += red[w];
    return total * p.num_hg;
}

// One segment: chunks [c0, c1) of (cur.b, cur.hg) inside unit u, or (dyn_t
// >= 0) the dynamic tail of (cur.b, cur.hg) handed out as ticket dyn_t.
struct Segment {
    Cursor cur;
    int c0, c1;
    long long u;        // unit (static segments)
    long long gstart;   // static-list index of chunk 0 of (b, hg) (static segments)
    int dyn_t;          // ticket of a dynamic tail, -1 for a static segment
};

// The r-th (0-based) request whose pass has at least one chunk; warp
// cooperative, every lane gets the result.  Returns false if there is none.
template <int CH>
__device__ bool nth_nonempty(const DecodeParams& p, long long r, int lane, Cursor& cur) {
    long long base = 0;
    for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
        const int b = b0 + lane;
        int L = 0, T = 0;
        if (b < p.num_seqs) {
            L = clamp_len(p, b, false);
            T = seq_begin(p, b, L);
        }
        const unsigned has = __ballot_sync(FULL_MASK, chunks_of<CH>(L - T) > 0);
        const long long cnt = __popc(has);
        if (r < base + cnt) {
            // the (r - base)-th set bit of `has`
            unsigned m = has;
            for (long long k = r - base; k > 0; --k) m &= m - 1;
            const int src = __ffs(m) - 1;
            cur.b = b0 + src;
            cur.L = __shfl_sync(FULL_MASK, L, src);
            cur.t0 = __shfl_sync(FULL_MASK, T, src);
            return true;
        }
        base += cnt;
    }
    return false;
}

// Static-list index of chunk 0 of (b, hg): the static chunks of the requests
// before b, all head groups, plus hg of request b's.  Warp cooperative.
template <int CH>
__device__ long long static_start(const DecodeParams& p, int b, int hg, int nch_static, int lane) {
    long long sum = 0;
    for (int b1 = lane; b1 < b; b1 += 32) {
        const int L = clamp_len(p, b1, false);
        sum += list_chunks<CH>(p, L - seq_begin(p, b1, L));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(FULL_MASK, sum, off);
    return sum * p.num_hg + (long long)hg * nch_static;
}

// Shared-memory queue of the dynamic tails a CTA takes: the fetching warp
// draws tickets from the workspace counter and publishes them in order; every
// other warp of the CTA reads them in the same order.  A ticket < 0 ends the
// CTA's work.
constexpr int kTailQueue = 8;
struct TailQueue {
    int* val;         // [kTailQueue]
    uint64_t* full;   // [kTailQueue], count 1 (the fetcher)
    uint64_t* empty;  // [kTailQueue], count = readers
};

// Iterates this CTA's segments: its static units x, x + gridDim.x, ... of the
// static list, then (dynamic tails on) the tails it draws.
template <int CH>
struct SegIter {
    long long total, W, nunits;
    long long u, s1, g;
    Cursor cur;
    bool valid;
    int L_first = -1;  // this lane's length of request `lane` (first 32 requests)
    int T_first = 0;   // and the first token of its pass
    // dynamic tails
    long long n_tails = 0;  // tickets in all: one per (non-empty request, head group)
    TailQueue q{};
    bool fetcher = false;   // this warp draws the tickets (one warp per CTA)
    int qk = 0;             // tails taken so far
    int dyn_t = -1;         // ticket of the current tail segment
    bool failed = false;    // a bounded wait on the queue gave up

    __device__ void start_unit(const DecodeParams& p, int lane) {
        valid = u < nunits;
        if (valid) {
            const long long s0 = u * W;
            s1 = min(s0 + W, total);
            g = s0;
            cur = locate<CH>(p, s0, lane, L_first, T_first);
            valid = cur.nch > 0;
        }
        if (!valid && p.tail_chunks > 0) next_tail(p, lane);
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

    // The next dynamic tail of this CTA (or the end of its work).
    __device__ void next_tail(const DecodeParams& p, int lane) {
        int t = -1;
        const int slot = qk % kTailQueue;
        const uint32_t ph = (uint32_t)(qk / kTailQueue) & 1u;
        ++qk;
        if (lane == 0) {
            if (fetcher) {
                // the ticket words are workspace: the previous kernel in the
                // stream may still be using this workspace
                griddep_wait();
                if (failed || !mbar_wait(&q.empty[slot], ph ^ 1u, p.wait_ns)) {
                    failed = true;
                } else {
                    t = (int)atomicAdd(p.tickets, 1u);
                    if (t >= n_tails) {
                        t = -1;
                        // the last CTA to run out returns both words to zero
                        if (atomicAdd(p.tickets + 1, 1u) == gridDim.x - 1) {
                            p.tickets[0] = 0u;
                            p.tickets[1] = 0u;
                        }
                    }
                }
                q.val[slot] = t;
                mbar_arrive(&q.full[slot]);
            } else {
                if (failed || !mbar_wait(&q.full[slot], ph, p.wait_ns)) {
                    failed = true;
                } else {
                    t = q.val[slot];
                    mbar_arrive(&q.empty[slot]);
                }
            }
            if (failed) raise_error(p.err, PKV_DEVERR_TIMEOUT);
        }
        t = __shfl_sync(FULL_MASK, t, 0);
        failed = __shfl_sync(FULL_MASK, failed ? 1 : 0, 0) != 0;
        dyn_t = t;
        valid = t >= 0 && nth_nonempty<CH>(p, t / p.num_hg, lane, cur);
        if (!valid) return;
        cur.hg = t % p.num_hg;
        cur.nch = chunks_of<CH>(cur.L - cur.t0);
        cur.c = max(cur.nch - p.tail_chunks, 0);
        g = 0;
        s1 = cur.nch - cur.c;
        u = -1;
    }

    __device__ __forceinline__ Segment current() const {
        Segment s;
        s.cur = cur;
        s.c0 = cur.c;
        s.c1 = (int)min((long long)cur.nch, (long long)cur.c + (s1 - g));
        s.u = u;
        s.gstart = g - cur.c;
        s.dyn_t = dyn_t;
        return s;
    }

    __device__ void advance(const DecodeParams& p, int lane) {
        const Segment s = current();
        g += s.c1 - s.c0;
        if (dyn_t >= 0) {
            next_tail(p, lane);
        } else if (g < s1) {
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
