// decode_prefix.cu -- the shared pass of prefix-aware paged decode, on the
// 5th-generation tensor cores (tcgen05, accumulators in tensor memory).
//
// Requests forked from one prompt share the physical blocks of its prefix
// ("KV Cache Management", "The Bonus: Zero-Copy Sharing"; "KV Cache
// Optimization and PagedAttention", intro: shared blocks are computed and
// stored once).  Decoding them one request at a time still reads those blocks
// once per request.  This pass reads each prefix tile once per 128 (member,
// query head) rows instead, which turns the group's decode over the prefix
// into a dense contraction with the rows as the MMA M dimension:
//   S[128 x 64] = Q[128 x d] . K_chunk^T     (tcgen05.mma, both operands K-major)
//   O[128 x d] += P[128 x 64] . V_chunk      (P K-major, V MN-major)
// S (two buffers) and O live in tensor memory: 64 + 64 + d columns of fp32
// over 128 lanes, one lane per row.  One thread of the MMA warp issues the
// MMAs; four softmax warps (one per 32-lane quarter of tensor memory, one row
// per thread) read S with tcgen05.ld, mask it, run the online softmax in base
// 2 and write P, split into bf16 hi + lo, back into the S buffer it came from
// (hi in its first 32 columns, lo in the next 32, two bf16 per column), where
// the P.V MMA reads it as its A operand (no shared-memory P, no store and
// proxy fence per chunk); the MMAs of one thread execute in order, so the next
// S into that buffer follows the P.V that reads it.  The running maximum is raised
// lazily: O (in tensor memory) is rescaled only when a row's maximum grows by
// more than 8 (a factor 256), so the weights stay below 2^8 and the result is
// exact whatever maximum is used, as long as O and the row sum l use the same.
//
// The pass leaves, per (split, request, query head), the partial state (max m
// in log2 units, sum l, unnormalised acc) of the attention over that split's
// prefix tokens; the per-request decode pass starts after the prefix and
// merges these states into its own:
//   out = (A + sum_s 2^(m_s - M) acc_s) / (S + sum_s 2^(m_s - M) l_s).
// A member shorter than the prefix has its row masked past its own length.
//
// Data movement as in the per-request decode kernel: a producer warp reads the
// block table of the group's longest member and issues TMA tensor copies
// (128-byte swizzle, no multicast) of each block's K and V rows of one kv head
// into a 3-stage ring; the stage is released by the MMA completion of the
// P.V product that reads it (tcgen05.commit on the stage's empty barrier).
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "decode_common.cuh"
#include "mma_ptx.cuh"
#include "umma_ptx.cuh"

namespace pkv {
namespace {

constexpr int kStagesP = 3;
constexpr int kSoftWarps = 4;                       // one row per thread
constexpr int kThreadsP = 32 * (2 + kSoftWarps);    // producer, MMA, softmax
constexpr int kTmemCols = 256;                      // S x2 (64 each) + O (<= 128)
constexpr int kSCol = 0, kOCol = 128;               // tensor-memory columns
static_assert(kSoftWarps * 32 == kPrefixRows, "one tile row per softmax thread");

template <int D>
struct PCfg {
    static constexpr int NHALF = D / 64;               // 128-byte halves of a bf16 row
    static constexpr int KS = D / 16;                  // k-steps of Q.K^T
    static constexpr int HALF_BYTES = kPrefixCH * 128; // one 64-column half of a K or V tile
    static constexpr int KV_BYTES = NHALF * HALF_BYTES;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;   // K | V, whole KB
    static constexpr int QHALF = kPrefixRows * 128;    // one 64-column half of the Q tile
    static constexpr int OFF_Q = kStagesP * STAGE_BYTES;
    static constexpr int OFF_BAR = OFF_Q + NHALF * QHALF;
    // full, empty per stage; s_full, s_free, p_full, pv_done per buffer; q_ready; drain
    static constexpr int NBAR = 2 * kStagesP + 4 * 2 + 2;
    static constexpr int OFF_META = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ROWS = OFF_META + 2 * kStagesP * 4;
    static constexpr int OFF_CTRL = OFF_ROWS + 3 * kPrefixRows * 4;
    static constexpr int BYTES = OFF_CTRL + 32 + 1024;  // + alignment slack
    static_assert(BYTES * kPrefixCtasPerSm <= 227 * 1024, "kPrefixCtasPerSm CTAs per SM");
};

// Instruction descriptors: S = Q.K^T (M 128, N 64, B K-major) and
// O += P.V (M 128, N d, B MN-major).
template <int D>
struct PIdesc {
    static constexpr uint32_t S = idesc_bf16_f32(kPrefixRows, kPrefixCH, false);
    static constexpr uint32_t PV = idesc_bf16_f32(kPrefixRows, D, true);
};

// Byte offset of the 16-byte chunk `c` (8 bf16) of row `r` in a 128-byte
// swizzled region (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

template <int D>
__global__ void __launch_bounds__(kThreadsP, kPrefixCtasPerSm)
    prefix_kernel(const __grid_constant__ PrefixParams p, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv) {
    using C = PCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + kStagesP;
    uint64_t* s_full = empty + kStagesP;  // S buffer b holds a chunk's scores
    uint64_t* s_free = s_full + 2;        // the softmax warps have read S buffer b
    uint64_t* p_full = s_free + 2;        // P in S buffer b (and any O rescale) is ready
    uint64_t* pv_done = p_full + 2;       // the P.V MMAs reading S buffer b's P completed
    uint64_t* q_ready = pv_done + 2;      // the Q tile is in shared memory
    uint64_t* drain = q_ready + 1;        // every MMA this CTA issued has completed
    int* st_ntok = reinterpret_cast<int*>(smem + C::OFF_META);
    unsigned* st_bad = reinterpret_cast<unsigned*>(st_ntok + kStagesP);
    int* row_b = reinterpret_cast<int*>(smem + C::OFF_ROWS);
    int* row_h = row_b + kPrefixRows;
    int* row_L = row_h + kPrefixRows;
    volatile int* ctrl = reinterpret_cast<volatile int*>(smem + C::OFF_CTRL);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_CTRL + 16);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    int x = blockIdx.x;
    const int sp = x % p.splits;
    x /= p.splits;
    const int rt = x % p.row_tiles;
    x /= p.row_tiles;
    const int kvh = x % p.num_kv_heads;
    const int g = x / p.num_kv_heads;
    const bool leader = sp == 0 && rt == 0 && kvh == 0;  // reports the group's errors once

    const int cap = p.max_blocks * p.block_size;
    const int ptok = prefix_tokens(p.prefix_lens, g, p.max_prefix_len, cap, p.log2_bs, p.err,
                                   leader && threadIdx.x == 0);
    const int nsplit = prefix_num_splits(ptok, p.splits);
    if (sp >= nsplit) {  // this split holds no chunk of the prefix
        // still wait for the previous kernel, so that this grid's completion
        // implies that kernel's (the decode pass after it relies on that)
        griddep_wait();
        return;
    }
    const int span = prefix_chunk_span(ptok, p.splits);
    const int nch = chunks_of<kPrefixCH>(ptok);
    const int c0 = sp * span, c1 = min(c0 + span, nch);

    if (threadIdx.x == 0) {
        ctrl[0] = 0;
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);  // the MMA completion of the chunk's P.V
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], kSoftWarps);
            mbar_init(&p_full[b], kSoftWarps * 32);
            mbar_init(&pv_done[b], 1);
        }
        mbar_init(q_ready, kSoftWarps * 32);
        mbar_init(drain, 1);
        fence_mbar_init();
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
    }
    if (warp == 1) {  // this warp owns the tensor memory: allocates and frees it
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    // Members of group g in request order; rank r holds rows r*G .. r*G+G-1.
    // The table source is the longest member (the first of equal ones).
    if (warp == 0) {
        for (int r = lane; r < kPrefixRows; r += 32) {
            row_b[r] = -1;
            row_h[r] = 0;
            row_L[r] = 0;
        }
        __syncwarp();
        const int r_lo = rt * kPrefixRows;
        int count = 0, best_L = -1, best_b = 0x7fffffff;
        auto scan = [&](int b0, int gb, int L) {
            const int b = b0 + lane;
            const bool mem = b < p.num_seqs && gb == g;
            const unsigned bal = __ballot_sync(FULL_MASK, mem);
            if (mem) {
                const int rank = count + __popc(bal & ((1u << lane) - 1u));
                L = L < 0 ? 0 : (L > cap ? cap : L);  // the decode pass flags it
                if (L > best_L) {
                    best_L = L;
                    best_b = b;
                }
                for (int j = 0; j < p.group; ++j) {
                    const int r = rank * p.group + j - r_lo;
                    if (r >= 0 && r < kPrefixRows) {
                        row_b[r] = b;
                        row_h[r] = kvh * p.group + j;
                        row_L[r] = L;
                    }
                }
            }
            count += __popc(bal);
        };
        // The first 128 requests' group ids and lengths are loaded together
        // (one round trip), the rest as the scan reaches them.
        constexpr int kAhead = 4;
        int gb[kAhead], lb[kAhead];
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
            const int b = 32 * k + lane;
            gb[k] = b < p.num_seqs ? __ldg(p.prefix_of + b) : -1;
            lb[k] = b < p.num_seqs ? __ldg(p.seq_lens + b) : 0;
        }
#pragma unroll
        for (int k = 0; k < kAhead; ++k)
            if (32 * k < p.num_seqs) scan(32 * k, gb[k], lb[k]);
        for (int b0 = 32 * kAhead; b0 < p.num_seqs; b0 += 32) {
            const int b = b0 + lane;
            scan(b0, b < p.num_seqs ? __ldg(p.prefix_of + b) : -1,
                 b < p.num_seqs ? __ldg(p.seq_lens + b) : 0);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const int oL = __shfl_xor_sync(FULL_MASK, best_L, off);
            const int ob = __shfl_xor_sync(FULL_MASK, best_b, off);
            if (oL > best_L || (oL == best_L && ob < best_b)) {
                best_L = oL;
                best_b = ob;
            }
        }
        if (lane == 0) {
            ctrl[1] = best_L < 0 ? -1 : best_b;
            ctrl[2] = best_L < 0 ? 0 : min(ptok, best_L);  // tokens anyone attends to
            ctrl[3] = count * p.group > r_lo;              // this tile has rows
            if (leader && count > p.max_members) raise_error(p.err, PKV_DEVERR_PREFIX);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    const uint32_t tmem = *tmem_slot;
    const int b_src = ctrl[1];
    const int tl = ctrl[2];
    const int c_end = ctrl[3] ? min(c1, chunks_of<kPrefixCH>(tl)) : c0;
    const int n_local = max(c_end - c0, 0);  // chunks this CTA streams

    if (warp == 0) {
        // ---- producer ----
        const uint64_t policy = l2_policy_evict_last();
        const int rb = min(p.block_size, kPrefixCH);
        const uint32_t stage_tx_per_block = 2u * rb * C::NHALF * 128u;
        const int32_t* table = p.block_tables + (size_t)max(b_src, 0) * p.max_blocks;
        Ring ring;
        int issued = 0;
        bool waited = false;
        auto window = [&](int c) {
            const int t0 = c * kPrefixCH;
            const int ja = t0 >> p.log2_bs;
            const int jb = (min(t0 + kPrefixCH, tl) - 1) >> p.log2_bs;
            return (c < c_end && lane <= jb - ja) ? __ldg(table + ja + lane) : -1;
        };
        int tab = window(c0);
        for (int c = c0; c < c_end; ++c) {
            const int tab_next = window(c + 1);
            const int t0 = c * kPrefixCH;
            const int ntok = min(kPrefixCH, tl - t0);
            const int ja = t0 >> p.log2_bs;
            const int jb = (t0 + ntok - 1) >> p.log2_bs;
            int ok = 1;
            if (lane == 0) ok = !ctrl[0] && mbar_wait(&empty[ring.stage], ring.phase ^ 1u);
            ok = __shfl_sync(FULL_MASK, ok, 0);
            if (!ok) {
                if (lane == 0) {
                    ctrl[0] = 1;
                    raise_error(p.err, PKV_DEVERR_TIMEOUT);
                }
                break;
            }
            if (!waited) {
                griddep_wait();  // the caches may come from the previous kernel
                waited = true;
            }
            uint32_t nvalid = 0, bad = 0;
            for (int j = ja; j <= jb; ++j) {
                const int phys = __shfl_sync(FULL_MASK, tab, j - ja);
                if (phys < 0 || phys >= p.num_blocks)
                    bad |= 1u << (j - ja);
                else
                    ++nvalid;
            }
            if (lane == 0) {
                st_ntok[ring.stage] = ntok;
                st_bad[ring.stage] = bad;
                if (bad) raise_error(p.err, PKV_DEVERR_BAD_BLOCK);
                mbar_arrive_expect_tx(&full[ring.stage], nvalid * stage_tx_per_block);
            }
            unsigned char* sk = smem + ring.stage * C::STAGE_BYTES;
            unsigned char* sv = sk + C::KV_BYTES;
            // one lane per block issues that block's copies (a TMA issue costs
            // the issuing thread ~0.1 us; lane-parallel issue overlaps them)
            __syncwarp();  // the expect-tx above comes first
            {
                const int j = ja + lane;
                const int phys = __shfl_sync(FULL_MASK, tab, min(j, jb) - ja);
                if (j <= jb && phys >= 0 && phys < p.num_blocks) {
                    // t0 is a multiple of 64 and of block_size when block_size <= 64
                    const int srow = max((j << p.log2_bs) - t0, 0);
                    const int boff = max(t0 - (j << p.log2_bs), 0);
                    const int grow = (phys * p.num_kv_heads + kvh) * p.block_size + boff;
#pragma unroll
                    for (int h = 0; h < C::NHALF; ++h) {
                        tma_load_2d(sk + h * C::HALF_BYTES + srow * 128, &tmk, h * 64, grow,
                                    &full[ring.stage], policy);
                        tma_load_2d(sv + h * C::HALF_BYTES + srow * 128, &tmv, h * 64, grow,
                                    &full[ring.stage], policy);
                    }
                }
            }
            ++issued;
            ring.advance(kStagesP);
            tab = tab_next;
        }
        if (!waited) griddep_wait();
        if (ctrl[0] && lane == 0) {
            // a wait gave up: let this warp's copies land before the CTA exits
            const int n = min(issued, kStagesP);
            Ring r = ring;
            for (int i = 0; i < n; ++i) {
                if (r.stage == 0) {
                    r.stage = kStagesP - 1;
                    r.phase ^= 1u;
                } else {
                    --r.stage;
                }
                mbar_wait(&full[r.stage], r.phase);
            }
        }
        return;
    }

    if (warp == 1) {
        // ---- MMA issue (one thread) ----
        if (lane == 0 && n_local > 0) {
            const uint32_t qb = smem_addr(smem + C::OFF_Q);
            const uint32_t sb = smem_addr(smem);
            bool ok = mbar_wait(q_ready, 0);
            tc_fence_after();
            // S_i = Q . K_i^T into S buffer i % 2, once that buffer was read
            auto issue_s = [&](int i) -> bool {
                const int st = i % kStagesP, b = i & 1;
                if (!mbar_wait(&full[st], (i / kStagesP) & 1u) ||
                    !mbar_wait(&s_free[b], ((i >> 1) & 1u) ^ 1u))
                    return false;
                tc_fence_after();
                const uint32_t kb = sb + st * C::STAGE_BYTES;
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    const uint32_t off = (ks & 3) * 32;  // k-step inside the 128-byte atom
                    const uint64_t a = smem_desc_sw128(qb + (ks >> 2) * C::QHALF + off, 16, 1024);
                    const uint64_t bd = smem_desc_sw128(kb + (ks >> 2) * C::HALF_BYTES + off, 16, 1024);
                    umma_bf16(tmem + kSCol + b * kPrefixCH, a, bd, PIdesc<D>::S, ks > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[b]);
                return true;
            };
            if (ok) ok = issue_s(0);
            for (int i = 0; i < n_local && ok; ++i) {
                const int st = i % kStagesP, b = i & 1;
                if (i + 1 < n_local && !issue_s(i + 1)) {  // overlaps the softmax of chunk i
                    ok = false;
                    break;
                }
                if (ctrl[0] || !mbar_wait(&p_full[b], (i >> 1) & 1u)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vb = sb + st * C::STAGE_BYTES + C::KV_BYTES;
#pragma unroll
                for (int part = 0; part < 2; ++part) {  // P hi, then P lo
                    // P of chunk i: columns [32 part, 32 part + 32) of S buffer b,
                    // 16 tokens (8 columns) per MMA
                    const uint32_t pa = tmem + kSCol + b * kPrefixCH + part * (kPrefixCH / 2);
#pragma unroll
                    for (int kt = 0; kt < kPrefixCH / 16; ++kt) {
                        const uint64_t bd = smem_desc_sw128(vb + kt * 16 * 128, C::HALF_BYTES, 1024);
                        const uint32_t acc = (i == 0 && part == 0 && kt == 0) ? 0u : 1u;
                        umma_bf16_ts(tmem + kOCol, pa + kt * 8, bd, PIdesc<D>::PV, acc);
                    }
                }
                umma_commit(&empty[st]);   // the K/V stage may be refilled
                umma_commit(&pv_done[b]);  // P buffer b may be rewritten; O is current
            }
            if (!ok) {
                if (!ctrl[0]) raise_error(p.err, PKV_DEVERR_TIMEOUT);
                ctrl[0] = 1;
            }
            // nothing may still write tensor memory when it is freed: a commit
            // tracks every MMA issued before it (bounded wait)
            umma_commit(drain);
            mbar_wait(drain, 0u);
        }
        __syncwarp();
    } else {
        // ---- softmax warps: thread t of warp w owns tile row 32 (w % 4) + t ----
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(quarter * 32) << 16);  // this warp's lanes
        const int b_r = row_b[r], h_r = row_h[r], L_r = row_L[r];
        griddep_wait();  // q may come from the previous kernel
        {
            // the row's q, bf16, into the swizzled K-major Q tile
            unsigned char* qs = smem + C::OFF_Q;
            const uint4* gq = reinterpret_cast<const uint4*>(
                static_cast<const __nv_bfloat16*>(p.q) + ((size_t)max(b_r, 0) * p.num_q_heads + h_r) * D);
#pragma unroll
            for (int c = 0; c < D / 8; ++c) {
                const uint4 v = b_r >= 0 ? __ldg(gq + c) : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4*>(qs + (c >> 3) * C::QHALF + sw128(r, c & 7)) = v;
            }
            fence_proxy_async_smem();  // generic writes -> the tensor cores' reads
            mbar_arrive(q_ready);
        }
        const float sl2 = p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        for (int i = 0; i < n_local; ++i) {
            const int st = i % kStagesP, b = i & 1, c = c0 + i;
            // the stage's token count (written before its copies), then the
            // scores.  Every decision before a tcgen05.ld/st is taken by the
            // whole warp (those instructions need all 32 lanes).
            bool ok = !ctrl[0] && mbar_wait(&full[st], (i / kStagesP) & 1u) &&
                      mbar_wait(&s_full[b], (i >> 1) & 1u);
            if (!__all_sync(FULL_MASK, ok)) {
                if (lane == 0 && !ctrl[0]) {
                    ctrl[0] = 1;
                    raise_error(p.err, PKV_DEVERR_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            float s[kPrefixCH];
            {
                // both 32-column halves in flight before one wait
                uint32_t u0[32], u1[32];
                tmem_ld32(trow + kSCol + b * kPrefixCH, u0);
                tmem_ld32(trow + kSCol + b * kPrefixCH + 32, u1);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    s[j] = __uint_as_float(u0[j]);
                    s[32 + j] = __uint_as_float(u1[j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[b]);

            const int ntok = st_ntok[st];
            const unsigned bad = st_bad[st];
            const bool whole = ntok == kPrefixCH && bad == 0;
            const int tbase = c * kPrefixCH;
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < kPrefixCH; ++j) {
                bool ok = tbase + j < L_r;
                if (!whole) {
                    const int jrel = ((tbase + j) >> p.log2_bs) - (tbase >> p.log2_bs);
                    ok = ok && j < ntok && !((bad >> jrel) & 1u);
                }
                s[j] = ok ? s[j] * sl2 : -INFINITY;
                mx = fmaxf(mx, s[j]);
            }
            // lazy maximum: raise it (and rescale O, l) only past a factor 2^8
            const bool raise = mx > m_used + 8.f;
            const float m_new = raise ? mx : m_used;
            if (__any_sync(FULL_MASK, raise) && i > 0) {
                const float alpha = raise ? exp2f(m_used - m_new) : 1.f;  // 0 from -inf
                // O must hold the previous chunk's P.V before it is rescaled
                if (!__all_sync(FULL_MASK, mbar_wait(&pv_done[(i - 1) & 1], ((i - 1) >> 1) & 1u))) {
                    if (lane == 0 && !ctrl[0]) {
                        ctrl[0] = 1;
                        raise_error(p.err, PKV_DEVERR_TIMEOUT);
                    }
                    break;
                }
                tc_fence_after();
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t u[32];
                    tmem_ld32(trow + kOCol + q * 32, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(__uint_as_float(u[j]) * alpha);
                    tmem_st32(trow + kOCol + q * 32, u);
                }
                tmem_wait_st();
                l *= alpha;
            }
            m_used = m_new;
            const float ref = m_used == -INFINITY ? 0.f : m_used;
            // P into S buffer b (its scores are in registers): hi in columns
            // [0, 32), lo in [32, 64), two tokens per column, 32 tokens at a time
            const uint32_t pcol = trow + kSCol + b * kPrefixCH;
#pragma unroll
            for (int hq = 0; hq < 2; ++hq) {
                uint32_t wh[16], wl[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = ex2_ftz(s[hq * 32 + 2 * e] - ref);
                    const float p1 = ex2_ftz(s[hq * 32 + 2 * e + 1] - ref);
                    l += p0 + p1;
                    const float h0 = bf16_round(p0), h1 = bf16_round(p1);
                    wh[e] = pack_bf16(h0, h1);
                    wl[e] = pack_bf16(p0 - h0, p1 - h1);
                }
                tmem_st16(pcol + hq * 16, wh);
                tmem_st16(pcol + kPrefixCH / 2 + hq * 16, wl);
            }
            tmem_wait_st();
            if (!whole) {
                // V rows of tokens that do not take part (past the chunk's end or
                // in a bad block) hold stale or poisoned data: zero them so that
                // 0-weight x NaN cannot reach O
                unsigned char* sv = smem + st * C::STAGE_BYTES + C::KV_BYTES;
                for (int idx = r; idx < kPrefixCH * C::NHALF * 8; idx += kPrefixRows) {
                    const int row = idx / (C::NHALF * 8), rest = idx % (C::NHALF * 8);
                    const int jrel = ((tbase + row) >> p.log2_bs) - (tbase >> p.log2_bs);
                    if (row >= ntok || ((bad >> jrel) & 1u))
                        *reinterpret_cast<uint4*>(sv + (rest >> 3) * C::HALF_BYTES + row * 128 +
                                                  (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            if (!whole) fence_proxy_async_smem();  // zeroed V rows -> the tensor cores' reads
            tc_fence_before();
            mbar_arrive(&p_full[b]);
        }
        // the partial state of this split for row r (an empty state when the
        // split holds no token that any member attends to)
        if (n_local == 0 && b_r >= 0) {
            const size_t row = ((size_t)sp * p.num_seqs + b_r) * p.num_q_heads + h_r;
            float4* ra = reinterpret_cast<float4*>(p.pfx_acc + row * D);
            for (int j = 0; j < D / 4; ++j) ra[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            p.pfx_ml[row * 2] = -INFINITY;
            p.pfx_ml[row * 2 + 1] = 0.f;
        }
        if (__all_sync(FULL_MASK, n_local > 0 && !ctrl[0])) {
            const int last = n_local - 1;
            if (__all_sync(FULL_MASK, mbar_wait(&pv_done[last & 1], (last >> 1) & 1u))) {
                tc_fence_after();
                float* ra = b_r >= 0 ? p.pfx_acc + (((size_t)sp * p.num_seqs + b_r) * p.num_q_heads + h_r) * D
                                     : nullptr;
#pragma unroll 1
                for (int q = 0; q < D / 32; ++q) {
                    uint32_t u[32];
                    tmem_ld32(trow + kOCol + q * 32, u);
                    tmem_wait_ld();
                    if (ra) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4)
                            *reinterpret_cast<float4*>(ra + q * 32 + j) =
                                make_float4(__uint_as_float(u[j]), __uint_as_float(u[j + 1]),
                                            __uint_as_float(u[j + 2]), __uint_as_float(u[j + 3]));
                    }
                }
                if (ra) {
                    const size_t row = ((size_t)sp * p.num_seqs + b_r) * p.num_q_heads + h_r;
                    p.pfx_ml[row * 2] = m_used;
                    p.pfx_ml[row * 2 + 1] = l;
                }
            } else if (lane == 0 && !ctrl[0]) {
                ctrl[0] = 1;
                raise_error(p.err, PKV_DEVERR_TIMEOUT);
            }
        }
        tc_fence_before();
    }
    // The MMA warp (its MMAs drained) and the softmax warps (their tensor-memory
    // loads and stores complete) meet before the tensor memory is freed.
    named_bar_sync(1, 32 * (1 + kSoftWarps));
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int D>
pkv_status launch_impl(const PrefixParams& p, const void* k_cache, const void* v_cache,
                       cudaStream_t stream) {
    using C = PCfg<D>;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    static std::mutex mu;
    static bool ready[64] = {false};
    auto kern = prefix_kernel<D>;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (di->device >= 64) return PKV_ERR_UNSUPPORTED;
        if (!ready[di->device]) {
            if (C::BYTES > di->max_smem_optin) return PKV_ERR_UNSUPPORTED;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::BYTES) !=
                cudaSuccess)
                return PKV_ERR_CUDA;
            ready[di->device] = true;
        }
    }
    const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
    const int box_rows = std::min(p.block_size, kPrefixCH);
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, k_cache, rows, D, box_rows, false) ||
        !encode_cache_map(&tmv, v_cache, rows, D, box_rows, false))
        return PKV_ERR_CUDA;
    const long long grid =
        (long long)p.num_prefixes * p.num_kv_heads * p.row_tiles * p.splits;
    if (grid <= 0) return PKV_OK;
    if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
    PdlLaunch L(dim3((unsigned)grid), dim3(kThreadsP), C::BYTES, stream);
    if (cudaLaunchKernelEx(&L.cfg, kern, p, tmk, tmv) != cudaSuccess) return PKV_ERR_CUDA;
    return PKV_OK;
}

}  // namespace

pkv_status launch_decode_prefix(const PrefixParams& p, const void* k_cache, const void* v_cache,
                                int head_dim, cudaStream_t stream) {
    if (head_dim == 128) return launch_impl<128>(p, k_cache, v_cache, stream);
    if (head_dim == 64) return launch_impl<64>(p, k_cache, v_cache, stream);
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace pkv
