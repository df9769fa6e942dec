// decode_simt.cu -- paged decode attention on the CUDA cores (fp32 math).
//
// What it computes ("PagedAttention: Optimizing KV Cache Utilization in Large
// Language Models", "The Math: Block Attention Calculation", read as one
// softmax over the whole request): for request b and query head h,
//     out[b,h,:] = sum_t softmax_t(scale * q[b,h,:] . K_t) V_t,
// where K_t / V_t are found through the request's block table ("The Mechanics
// of PagedAttention": logical block -> physical block, like an OS page table).
//
// Decomposition (flash-decoding style split over the sequence):
//   * The work of one call is the flattened list of 32-token chunks over
//     (request b, head group hg, chunk c); a head group is one kv head and the
//     (up to 8) query heads that read it, so each K/V tile is read once per kv
//     head.  The list is cut into equal units of W chunks; a persistent grid
//     (SM count x resident CTAs) walks the units, so every CTA streams the same
//     number of bytes whatever the length mix.
//   * A unit is processed as segments (maximal runs inside one (b, hg)).  A
//     segment that covers a whole (b, hg) writes the normalised output
//     directly; otherwise it writes a partial record (running max, normaliser,
//     un-normalised weighted V sum) and the merge kernel combines the records:
//         out = sum_u 2^(m_u - M) acc_u / sum_u 2^(m_u - M) l_u,  M = max_u m_u.
//
// CTA = 1 producer warp + 4 consumer warps.
//   * Producer: walks the block table (32 entries per coalesced load, held in
//     lane registers), and for each chunk issues bulk TMA copies
//     (cp.async.bulk, no multicast) of the K and V rows of each physical block
//     into a ring of shared-memory stages, completing on a per-stage mbarrier.
//   * Consumers: each takes 8 of a stage's 32 tokens.  A token is spread over
//     LPT lanes, each holding DPL dims of q (pre-scaled by scale*log2 e, in
//     registers) for all query heads of the group; q.K partials are summed with
//     xor-shuffles, the softmax runs online per lane (base 2), and the P.V
//     update accumulates into the same lane's dims.  Lanes/warps are merged once
//     per segment (shuffles, then shared memory).
#include <algorithm>
#include <mutex>

#include "decode_common.cuh"

namespace pkv {
namespace {

constexpr int kChunk = 32;         // tokens per pipeline stage
constexpr int kConsumerWarps = 4;  // consumer warps per CTA
constexpr int kThreads = 32 * (1 + kConsumerWarps);
constexpr int kRingBudget = 81920;  // bytes of K/V stages per CTA

constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int align_up(int x, int a) { return (x + a - 1) / a * a; }

template <typename KV, int D, int GP>
struct SimtCfg {
    static constexpr int ES = Elem<KV>::kBytes;
    static constexpr int EPV = Elem<KV>::kPerVec;             // elements per 16 B
    static constexpr int TOKW = kChunk / kConsumerWarps;      // tokens per warp per stage
    static constexpr int DPL = cmin(cmin(64 / GP, 32), D / 4);  // dims per lane
    static constexpr int LPT = D / DPL;                       // lanes per token
    static constexpr int TPW = 32 / LPT;                      // tokens per pass
    static constexpr int PASSES = TOKW / TPW;
    static constexpr int NV = DPL / EPV;                      // 16-B vectors per lane per row
    static constexpr int ROW_BYTES = D * ES;
    static constexpr int HALF_BYTES = kChunk * ROW_BYTES;     // K (or V) part of a stage
    static constexpr int STAGE_BYTES = 2 * HALF_BYTES;
    static constexpr int NSTAGE = cmax(2, cmin(8, kRingBudget / STAGE_BYTES));
    static constexpr int OFF_BAR = NSTAGE * STAGE_BYTES;
    static constexpr int OFF_META = OFF_BAR + 2 * NSTAGE * 8;
    static constexpr int OFF_RED = align_up(OFF_META + 2 * NSTAGE * 4, 128);
    static constexpr int OFF_REDML = OFF_RED + kConsumerWarps * GP * D * 4;
    static constexpr int OFF_SCRATCH = align_up(OFF_REDML + kConsumerWarps * GP * 2 * 4, 16);
    static constexpr int OFF_CTRL = OFF_SCRATCH + 16 * 8;  // abort flag, stages issued
    static constexpr int SMEM = OFF_CTRL + 16;
    static_assert(TPW * LPT == 32 && PASSES * TPW == TOKW, "lane mapping");
    static_assert(NV >= 1 && NV * EPV == DPL, "vector mapping");
    static_assert(ROW_BYTES % 16 == 0, "rows must be whole 16-byte vectors");
};

__device__ __forceinline__ int chunks_of_len(int L) { return chunks_of<kChunk>(L); }

__device__ __forceinline__ Cursor locate(const DecodeParams& p, long long s, int lane) {
    return pkv::locate<kChunk>(p, s, lane);
}

__device__ __forceinline__ void next_group(const DecodeParams& p, Cursor& cur) {
    pkv::next_group<kChunk>(p, cur);
}

template <typename KV, int D, int GP>
__device__ __forceinline__ void produce_segment(const DecodeParams& p, const Cursor& cur, int c0,
                                                int c1, unsigned char* smem, uint64_t* full,
                                                uint64_t* empty, int* st_ntok, unsigned* st_bad,
                                                Ring& ring, int lane, uint64_t policy,
                                                volatile int* ctrl) {
    using C = SimtCfg<KV, D, GP>;
    const int kvh = cur.hg / p.num_sub;
    const int nblk = (cur.L + p.block_size - 1) >> p.log2_bs;
    const int32_t* trow = p.block_tables + (size_t)cur.b * p.max_blocks;
    const unsigned char* kbase = static_cast<const unsigned char*>(p.k_cache);
    const unsigned char* vbase = static_cast<const unsigned char*>(p.v_cache);
    int wbase = -1, tab = -1;
    for (int c = c0; c < c1; ++c) {
        const int t0 = c * kChunk;
        const int ntok = cmin(kChunk, cur.L - t0);
        const int ja = t0 >> p.log2_bs;
        const int jb = (t0 + ntok - 1) >> p.log2_bs;
        if (wbase < 0 || ja >= wbase + 32) {
            wbase = ja & ~31;
            const int j = wbase + lane;
            tab = j < nblk ? __ldg(trow + j) : -1;
        }
        int ok = 1;
        if (lane == 0) ok = !ctrl[0] && mbar_wait(&empty[ring.stage], ring.phase ^ 1u);
        ok = __shfl_sync(FULL_MASK, ok, 0);
        if (!ok) {
            if (lane == 0) {
                ctrl[0] = 1;
                raise_error(p.err, PKV_DEVERR_TIMEOUT);
            }
            return;
        }
        uint32_t bytes = 0, bad = 0;
        for (int j = ja; j <= jb; ++j) {
            const int phys = __shfl_sync(FULL_MASK, tab, j - wbase);
            const int r0 = max(t0, j << p.log2_bs);
            const int r1 = min(t0 + ntok, (j + 1) << p.log2_bs);
            if (phys < 0 || phys >= p.num_blocks)
                bad |= 1u << (j - ja);
            else
                bytes += 2u * (uint32_t)(r1 - r0) * C::ROW_BYTES;
        }
        unsigned char* sk = smem + ring.stage * C::STAGE_BYTES;
        unsigned char* sv = sk + C::HALF_BYTES;
        if (lane == 0) {
            st_ntok[ring.stage] = ntok;
            st_bad[ring.stage] = bad;
            if (bad) raise_error(p.err, PKV_DEVERR_BAD_BLOCK);
            mbar_arrive_expect_tx(&full[ring.stage], bytes);
        }
        for (int j = ja; j <= jb; ++j) {
            const int phys = __shfl_sync(FULL_MASK, tab, j - wbase);
            if (lane == 0 && phys >= 0 && phys < p.num_blocks) {
                const int r0 = max(t0, j << p.log2_bs);
                const int r1 = min(t0 + ntok, (j + 1) << p.log2_bs);
                const size_t row0 =
                    ((size_t)phys * p.num_kv_heads + kvh) * p.block_size + (r0 - (j << p.log2_bs));
                const uint32_t nbytes = (uint32_t)(r1 - r0) * C::ROW_BYTES;
                const int dst = (r0 - t0) * C::ROW_BYTES;
                bulk_load(sk + dst, kbase + row0 * C::ROW_BYTES, nbytes, &full[ring.stage], policy);
                bulk_load(sv + dst, vbase + row0 * C::ROW_BYTES, nbytes, &full[ring.stage], policy);
            }
        }
        if (lane == 0) ctrl[1] = ctrl[1] + 1;  // stages issued so far
        ring.advance(C::NSTAGE);
    }
}

template <typename KV, int D, int GP>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(const __grid_constant__ DecodeParams p) {
    using C = SimtCfg<KV, D, GP>;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + C::NSTAGE;
    int* st_ntok = reinterpret_cast<int*>(smem + C::OFF_META);
    unsigned* st_bad = reinterpret_cast<unsigned*>(st_ntok + C::NSTAGE);
    float* red_acc = reinterpret_cast<float*>(smem + C::OFF_RED);
    float* red_ml = reinterpret_cast<float*>(smem + C::OFF_REDML);
    long long* scratch = reinterpret_cast<long long*>(smem + C::OFF_SCRATCH);
    volatile int* ctrl = reinterpret_cast<volatile int*>(smem + C::OFF_CTRL);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        ctrl[0] = 0;
        ctrl[1] = 0;
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }

    // Total chunk count of the call (the same in every CTA).
    long long local = 0;
    for (int b = threadIdx.x; b < p.num_seqs; b += kThreads)
        local += chunks_of_len(clamp_len(p, b, blockIdx.x == 0));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(FULL_MASK, local, off);
    if (lane == 0) scratch[warp] = local;
    __syncthreads();
    long long total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) total += scratch[w];
    total *= p.num_hg;
    if (total == 0) return;
    long long W = p.fixed_units > 0 ? p.fixed_units : (total + gridDim.x - 1) / gridDim.x;
    if (W < 1) W = 1;
    const long long nunits = (total + W - 1) / W;

    Ring ring;

    if (warp == 0) {
        // ---------------- producer ----------------
        const uint64_t policy = l2_policy_evict_first();
        for (long long u = blockIdx.x; u < nunits && !ctrl[0]; u += gridDim.x) {
            const long long s0 = u * W, s1 = min(s0 + W, total);
            Cursor cur = locate(p, s0, lane);
            long long g = s0;
            while (g < s1 && cur.nch > 0 && !ctrl[0]) {
                const int c0 = cur.c;
                const int c1 = (int)min((long long)cur.nch, c0 + (s1 - g));
                produce_segment<KV, D, GP>(p, cur, c0, c1, smem, full, empty, st_ntok, st_bad,
                                           ring, lane, policy, ctrl);
                g += c1 - c0;
                if (g < s1) next_group(p, cur);
            }
        }
        if (ctrl[0] && lane == 0) {
            // A wait gave up somewhere in the CTA.  Before this warp exits, wait
            // (bounded) for the last stages it issued, so no bulk copy can land
            // in shared memory after the CTA is gone.
            const int n = min(ctrl[1], C::NSTAGE);
            Ring r = ring;
            for (int i = 0; i < n; ++i) {
                if (r.stage == 0) {
                    r.stage = C::NSTAGE - 1;
                    r.phase ^= 1u;
                } else {
                    --r.stage;
                }
                mbar_wait(&full[r.stage], r.phase);
            }
        }
        return;
    }

    // ---------------- consumers ----------------
    const int cw = warp - 1;            // consumer warp index
    const int tt = lane / C::LPT;       // token lane-group within a pass
    const int kd = lane % C::LPT;       // dim slice
    const int ct = threadIdx.x - 32;    // consumer thread index
    constexpr int NCT = 32 * kConsumerWarps;

    for (long long u = blockIdx.x; u < nunits; u += gridDim.x) {
        const long long s0 = u * W, s1 = min(s0 + W, total);
        Cursor cur = locate(p, s0, lane);
        long long g = s0;
        while (g < s1 && cur.nch > 0) {
            const int c0 = cur.c;
            const int c1 = (int)min((long long)cur.nch, c0 + (s1 - g));
            const long long gstart = g - c0;  // global index of chunk 0 of (b, hg)
            const long long u_first = gstart / W;
            const long long u_last = (gstart + cur.nch - 1) / W;
            const int nseg = (int)(u_last - u_first + 1);
            const int kvh = cur.hg / p.num_sub;
            const int sub = cur.hg % p.num_sub;
            const int hq0 = kvh * p.group + sub * GP;
            const int gv = min(GP, p.group - sub * GP);
            const int bg = cur.b * p.num_hg + cur.hg;

            // q for the group's heads, this lane's dims, in the log2 domain.
            float qf[GP][C::DPL];
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                const KV* qrow = static_cast<const KV*>(p.q) +
                                 ((size_t)cur.b * p.num_q_heads + hq0 + (h < gv ? h : 0)) * D;
#pragma unroll
                for (int i = 0; i < C::NV; ++i) {
                    float f[C::EPV];
                    const uint4 v = __ldg(reinterpret_cast<const uint4*>(qrow) + kd + C::LPT * i);
                    Elem<KV>::unpack(v, f);
#pragma unroll
                    for (int e = 0; e < C::EPV; ++e)
                        qf[h][i * C::EPV + e] = h < gv ? f[e] * p.scale_log2 : 0.f;
                }
            }
            float m[GP], l[GP], acc[GP][C::DPL];
#pragma unroll
            for (int h = 0; h < GP; ++h) {
                m[h] = -INFINITY;
                l[h] = 0.f;
#pragma unroll
                for (int e = 0; e < C::DPL; ++e) acc[h][e] = 0.f;
            }

            for (int c = c0; c < c1; ++c) {
                // After any timeout the CTA stops waiting and only keeps its
                // named-barrier schedule, so no warp can be left behind.
                if (ctrl[0]) {
                    ring.advance(C::NSTAGE);
                    continue;
                }
                if (!mbar_wait(&full[ring.stage], ring.phase)) {
                    if (lane == 0) {
                        ctrl[0] = 1;
                        raise_error(p.err, PKV_DEVERR_TIMEOUT);
                    }
                    __syncwarp();
                    ring.advance(C::NSTAGE);
                    continue;
                }
                const int ntok = st_ntok[ring.stage];
                const unsigned bad = st_bad[ring.stage];
                const unsigned char* sk = smem + ring.stage * C::STAGE_BYTES;
                const unsigned char* sv = sk + C::HALF_BYTES;
                const int tw0 = cw * C::TOKW;
                const bool whole = (ntok == kChunk) && (bad == 0);

                float s[C::PASSES][GP];
#pragma unroll
                for (int ps = 0; ps < C::PASSES; ++ps) {
                    const int row = tw0 + ps * C::TPW + tt;
                    float kf[C::DPL];
#pragma unroll
                    for (int i = 0; i < C::NV; ++i) {
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            sk + row * C::ROW_BYTES + (kd + C::LPT * i) * 16);
                        Elem<KV>::unpack(v, kf + i * C::EPV);
                    }
#pragma unroll
                    for (int h = 0; h < GP; ++h) {
                        float a = 0.f;
#pragma unroll
                        for (int e = 0; e < C::DPL; ++e) a = fmaf(qf[h][e], kf[e], a);
                        s[ps][h] = a;
                    }
                }
#pragma unroll
                for (int off = 1; off < C::LPT; off <<= 1)
#pragma unroll
                    for (int ps = 0; ps < C::PASSES; ++ps)
#pragma unroll
                        for (int h = 0; h < GP; ++h)
                            s[ps][h] += __shfl_xor_sync(FULL_MASK, s[ps][h], off);

                bool valid[C::PASSES];
#pragma unroll
                for (int ps = 0; ps < C::PASSES; ++ps) {
                    valid[ps] = true;
                    if (!whole) {
                        const int t = tw0 + ps * C::TPW + tt;
                        const int jrel = ((c * kChunk + t) >> p.log2_bs) - ((c * kChunk) >> p.log2_bs);
                        valid[ps] = t < ntok && !((bad >> jrel) & 1u);
                        if (!valid[ps]) {
#pragma unroll
                            for (int h = 0; h < GP; ++h) s[ps][h] = -INFINITY;
                        }
                    }
                }

                // Online softmax, base 2, per lane.
                bool grew = false;
                float alpha[GP];
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    float mx = s[0][h];
#pragma unroll
                    for (int ps = 1; ps < C::PASSES; ++ps) mx = fmaxf(mx, s[ps][h]);
                    const float mnew = fmaxf(m[h], mx);
                    const float mref = mnew == -INFINITY ? 0.f : mnew;
                    grew |= mnew > m[h];
                    alpha[h] = exp2f(m[h] - mref);
                    m[h] = mnew;
                    float psum = 0.f;
#pragma unroll
                    for (int ps = 0; ps < C::PASSES; ++ps) {
                        s[ps][h] = exp2f(s[ps][h] - mref);
                        psum += s[ps][h];
                    }
                    l[h] = fmaf(l[h], alpha[h], psum);
                }
                if (__any_sync(FULL_MASK, grew)) {
#pragma unroll
                    for (int h = 0; h < GP; ++h)
#pragma unroll
                        for (int e = 0; e < C::DPL; ++e) acc[h][e] *= alpha[h];
                }

#pragma unroll
                for (int ps = 0; ps < C::PASSES; ++ps) {
                    const int row = tw0 + ps * C::TPW + tt;
                    float vf[C::DPL];
#pragma unroll
                    for (int i = 0; i < C::NV; ++i) {
                        const uint4 v = *reinterpret_cast<const uint4*>(
                            sv + row * C::ROW_BYTES + (kd + C::LPT * i) * 16);
                        Elem<KV>::unpack(v, vf + i * C::EPV);
                    }
                    if (!valid[ps]) {
#pragma unroll
                        for (int e = 0; e < C::DPL; ++e) vf[e] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < GP; ++h)
#pragma unroll
                        for (int e = 0; e < C::DPL; ++e) acc[h][e] = fmaf(s[ps][h], vf[e], acc[h][e]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[ring.stage]);
                ring.advance(C::NSTAGE);
            }

            // ---- merge the lanes that own different tokens (same dims) ----
#pragma unroll
            for (int off = C::LPT; off < 32; off <<= 1) {
#pragma unroll
                for (int h = 0; h < GP; ++h) {
                    const float mo = __shfl_xor_sync(FULL_MASK, m[h], off);
                    const float lo = __shfl_xor_sync(FULL_MASK, l[h], off);
                    const float M = fmaxf(m[h], mo);
                    const float mref = M == -INFINITY ? 0.f : M;
                    const float a = exp2f(m[h] - mref), bsc = exp2f(mo - mref);
                    l[h] = l[h] * a + lo * bsc;
                    m[h] = M;
#pragma unroll
                    for (int e = 0; e < C::DPL; ++e) {
                        const float ao = __shfl_xor_sync(FULL_MASK, acc[h][e], off);
                        acc[h][e] = acc[h][e] * a + ao * bsc;
                    }
                }
            }
            if (tt == 0) {
#pragma unroll
                for (int h = 0; h < GP; ++h) {
#pragma unroll
                    for (int i = 0; i < C::NV; ++i)
#pragma unroll
                        for (int e = 0; e < C::EPV; ++e)
                            red_acc[(cw * GP + h) * D + (kd + C::LPT * i) * C::EPV + e] =
                                acc[h][i * C::EPV + e];
                    if (kd == 0) {
                        red_ml[(cw * GP + h) * 2] = m[h];
                        red_ml[(cw * GP + h) * 2 + 1] = l[h];
                    }
                }
            }
            named_bar_sync(1, NCT);
            // ---- merge the consumer warps; write output or a partial record ----
            for (int idx = ct; idx < gv * D; idx += NCT) {
                const int h = idx / D, k = idx % D;
                float M = -INFINITY;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_ml[(w * GP + h) * 2]);
                const float mref = M == -INFINITY ? 0.f : M;
                float S = 0.f, A = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float f = exp2f(red_ml[(w * GP + h) * 2] - mref);
                    S = fmaf(red_ml[(w * GP + h) * 2 + 1], f, S);
                    A = fmaf(red_acc[(w * GP + h) * D + k], f, A);
                }
                if (nseg == 1) {
                    store_out(p.out, ((size_t)cur.b * p.num_q_heads + hq0 + h) * D + k,
                              S > 0.f ? A / S : 0.f, p.out_dtype);
                } else if ((long long)bg + u < p.rec_cap) {
                    const size_t rec = (size_t)bg + (size_t)u;
                    p.rec_acc[(rec * GP + h) * D + k] = A;
                    if (k == 0) {
                        p.rec_ml[(rec * GP + h) * 2] = M;
                        p.rec_ml[(rec * GP + h) * 2 + 1] = S;
                    }
                }
            }
            if (c0 == 0 && ct == 0) {
                // More units than the workspace was sized for (seq_lens above the
                // max_seq_len the caller declared): flag it, and mark the group so
                // the merge leaves its output alone instead of reading past the end.
                const bool fits = (long long)bg + u_last < p.rec_cap;
                if (!fits) raise_error(p.err, PKV_DEVERR_BAD_SEQ_LEN);
                p.meta[2 * (size_t)bg] = (int32_t)u;
                p.meta[2 * (size_t)bg + 1] = fits ? nseg : 0;
            }
            named_bar_sync(1, NCT);

            g += c1 - c0;
            if (g < s1) next_group(p, cur);
        }
    }
}

// Combine the partial records of every (request, head group) that was split
// over several units; write zeros for empty requests.
__global__ void decode_merge_kernel(const __grid_constant__ DecodeParams p, int GP, int D) {
    const int bg = blockIdx.x;
    const int b = bg / p.num_hg, hg = bg % p.num_hg;
    const int kvh = hg / p.num_sub, sub = hg % p.num_sub;
    const int hq0 = kvh * p.group + sub * GP;
    const int gv = min(GP, p.group - sub * GP);
    int L = __ldg(p.seq_lens + b);
    const int cap = p.max_blocks * p.block_size;
    L = L < 0 ? 0 : (L > cap ? cap : L);
    if (L == 0) {
        for (int idx = threadIdx.x; idx < gv * D; idx += blockDim.x)
            store_out(p.out, ((size_t)b * p.num_q_heads + hq0 + idx / D) * D + idx % D, 0.f,
                      p.out_dtype);
        return;
    }
    const int u0 = p.meta[2 * (size_t)bg];
    const int nseg = p.meta[2 * (size_t)bg + 1];
    if (nseg > 1) {
        for (int idx = threadIdx.x; idx < gv * D; idx += blockDim.x) {
            const int h = idx / D, k = idx % D;
            float M = -INFINITY;
            for (int r = 0; r < nseg; ++r) {
                const size_t rec = (size_t)bg + u0 + r;
                M = fmaxf(M, p.rec_ml[(rec * GP + h) * 2]);
            }
            const float mref = M == -INFINITY ? 0.f : M;
            float S = 0.f, A = 0.f;
            for (int r = 0; r < nseg; ++r) {
                const size_t rec = (size_t)bg + u0 + r;
                const float f = exp2f(p.rec_ml[(rec * GP + h) * 2] - mref);
                S = fmaf(p.rec_ml[(rec * GP + h) * 2 + 1], f, S);
                A = fmaf(p.rec_acc[(rec * GP + h) * D + k], f, A);
            }
            store_out(p.out, ((size_t)b * p.num_q_heads + hq0 + h) * D + k, S > 0.f ? A / S : 0.f,
                      p.out_dtype);
        }
    }
}

template <typename KV, int D, int GP>
pkv_status launch_impl(const DecodeParams& p, cudaStream_t stream, int* grid_out) {
    using C = SimtCfg<KV, D, GP>;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    static std::mutex mu;
    static int occupancy[64] = {0};
    auto kern = decode_simt_kernel<KV, D, GP>;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (di->device >= 64) return PKV_ERR_UNSUPPORTED;
        if (occupancy[di->device] == 0) {
            if (C::SMEM > di->max_smem_optin) return PKV_ERR_UNSUPPORTED;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) !=
                cudaSuccess)
                return PKV_ERR_CUDA;
            int occ = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kThreads, C::SMEM) !=
                    cudaSuccess ||
                occ < 1)
                return PKV_ERR_CUDA;
            occupancy[di->device] = occ;
        }
    }
    const int grid = di->num_sms * std::min(occupancy[di->device], 4);
    kern<<<grid, kThreads, C::SMEM, stream>>>(p);
    if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    decode_merge_kernel<<<p.num_seqs * p.num_hg, D, 0, stream>>>(p, GP, D);
    if (cudaGetLastError() != cudaSuccess) return PKV_ERR_CUDA;
    if (grid_out) *grid_out = grid;
    return PKV_OK;
}

template <typename KV, int D>
pkv_status dispatch_group(const DecodeParams& p, int group_pad, cudaStream_t s, int* g) {
    switch (group_pad) {
        case 1: return launch_impl<KV, D, 1>(p, s, g);
        case 2: return launch_impl<KV, D, 2>(p, s, g);
        case 4: return launch_impl<KV, D, 4>(p, s, g);
        case 8: return launch_impl<KV, D, 8>(p, s, g);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

}  // namespace

pkv_status launch_decode_simt(const DecodeParams& p, int head_dim, pkv_dtype kv_dtype,
                              int group_pad, cudaStream_t stream, int* grid_out) {
    if (kv_dtype == PKV_F32) {
        if (head_dim == 64) return dispatch_group<float, 64>(p, group_pad, stream, grid_out);
        if (head_dim == 128) return dispatch_group<float, 128>(p, group_pad, stream, grid_out);
    } else if (kv_dtype == PKV_BF16) {
        if (head_dim == 64) return dispatch_group<__nv_bfloat16, 64>(p, group_pad, stream, grid_out);
        if (head_dim == 128) return dispatch_group<__nv_bfloat16, 128>(p, group_pad, stream, grid_out);
    }
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace pkv
