// decode_prefix.cu -- the shared pass of prefix-aware paged decode.
//
// Requests forked from one prompt share the physical blocks of its prefix
// ("KV Cache Management", "The Bonus: Zero-Copy Sharing"; "KV Cache
// Optimization and PagedAttention", intro: shared blocks are computed and
// stored once).  Decoding them one request at a time still reads those blocks
// once per request.  This pass reads each prefix tile once per 64 (member,
// query head) rows instead, which turns the group's decode over the prefix
// into a dense contraction with the rows as the MMA M dimension:
//   S[64 x 64]  = Q[64 x d] . K_chunk^T       (q rows of 16 members x 4 heads)
//   O[64 x d]  += P[64 x 64] . V_chunk
// Each consumer warp owns 16 rows and runs the FlashAttention-2 register
// layout (Q as A fragments in registers, K via ldmatrix as the B operand, the
// S accumulator re-packed in registers as the A operand of P.V, V via
// ldmatrix.trans), online softmax in base 2 with P split into bf16 hi + lo.
//
// The pass leaves, per (split, request, query head), the partial state
// (max m in log2 units, sum l, unnormalised acc) of the attention over that
// split's prefix tokens; the per-request decode pass starts after the prefix
// and merges these states into its own:
//   out = (A + sum_s 2^(m_s - M) acc_s) / (S + sum_s 2^(m_s - M) l_s).
// A member shorter than the prefix has its rows masked past its own length.
//
// Data movement as in the per-request decode kernel: one producer warp reads
// the block table of the group's longest member and issues TMA tensor copies
// (128-byte swizzle, no multicast) of each block's K and V rows of one kv head
// into a 3-stage ring; the four consumer warps all read every stage.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "decode_common.cuh"
#include "mma_ptx.cuh"

namespace pkv {
namespace {

constexpr int kCW = 4;                     // consumer warps, 16 rows each
constexpr int kThreadsP = 32 * (1 + kCW);  // + the producer warp
constexpr int kStagesP = 3;
static_assert(kCW * 16 == kPrefixRows, "one row tile per CTA");

template <int D>
struct PCfg {
    static constexpr int NHALF = D / 64;               // 128-byte halves of a bf16 row
    static constexpr int KS = D / 16;                  // k-steps of Q.K^T
    static constexpr int DT = D / 8;                   // 8-wide output tiles
    static constexpr int HALF_BYTES = kPrefixCH * 128;
    static constexpr int KV_BYTES = NHALF * HALF_BYTES;
    static constexpr int STAGE_BYTES = 2 * KV_BYTES;   // K | V, whole KB
    static constexpr int OFF_BAR = kStagesP * STAGE_BYTES;
    static constexpr int OFF_META = OFF_BAR + 2 * kStagesP * 8;
    static constexpr int OFF_ROWS = OFF_META + 2 * kStagesP * 4;
    static constexpr int OFF_CTRL = OFF_ROWS + 3 * kPrefixRows * 4;
    static constexpr int BYTES = OFF_CTRL + 32 + 1024;  // + alignment slack
};

// smem address of the 16-byte chunk holding (row, col) of a swizzled tile
// region (rows of 128 bytes per 64-column half; chunk index XOR row % 8)
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int col, int half_bytes) {
    const int half = col >> 6, cc = (col & 63) >> 3;
    return base + half * half_bytes + row * 128 + ((cc ^ (row & 7)) << 4);
}

template <int D>
__global__ void __launch_bounds__(kThreadsP, 2)
    prefix_kernel(const __grid_constant__ PrefixParams p, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv) {
    using C = PCfg<D>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* empty = full + kStagesP;
    int* st_ntok = reinterpret_cast<int*>(smem + C::OFF_META);
    unsigned* st_bad = reinterpret_cast<unsigned*>(st_ntok + kStagesP);
    int* row_b = reinterpret_cast<int*>(smem + C::OFF_ROWS);
    int* row_h = row_b + kPrefixRows;
    int* row_L = row_h + kPrefixRows;
    volatile int* ctrl = reinterpret_cast<volatile int*>(smem + C::OFF_CTRL);
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
            mbar_init(&empty[s], kCW);
        }
        fence_mbar_init();
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
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
        for (int b0 = 0; b0 < p.num_seqs; b0 += 32) {
            const int b = b0 + lane;
            const bool mem = b < p.num_seqs && __ldg(p.prefix_of + b) == g;
            const unsigned bal = __ballot_sync(FULL_MASK, mem);
            if (mem) {
                const int rank = count + __popc(bal & ((1u << lane) - 1u));
                int L = __ldg(p.seq_lens + b);
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
    __syncthreads();
    griddep_launch_dependents();
    if (!ctrl[3]) {
        griddep_wait();
        return;
    }
    const int b_src = ctrl[1];
    const int tl = ctrl[2];
    const int c_end = min(c1, chunks_of<kPrefixCH>(tl));

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

    // ---- consumers: warp w owns rows 16w .. 16w+15 of the tile ----
    const int w = warp - 1;
    const int grp = lane >> 2, tig = lane & 3;
    const int rA = w * 16 + grp, rB = rA + 8;
    const int bA = row_b[rA], bB = row_b[rB];
    const int hA = row_h[rA], hB = row_h[rB];
    const int LA = row_L[rA], LB = row_L[rB];
    griddep_wait();  // q may come from the previous kernel

    // Q as A fragments: a0 = (row grp, k 2tig..+1), a1 = (row grp+8, ...),
    // a2 = (row grp, k 8+2tig..), a3 = (row grp+8, k 8+2tig..) per 16-wide k-step
    uint32_t qa[C::KS][4];
    {
        const uint32_t* qA = reinterpret_cast<const uint32_t*>(
            static_cast<const __nv_bfloat16*>(p.q) + ((size_t)max(bA, 0) * p.num_q_heads + hA) * D);
        const uint32_t* qB = reinterpret_cast<const uint32_t*>(
            static_cast<const __nv_bfloat16*>(p.q) + ((size_t)max(bB, 0) * p.num_q_heads + hB) * D);
#pragma unroll
        for (int ks = 0; ks < C::KS; ++ks) {
            qa[ks][0] = bA >= 0 ? __ldg(qA + ks * 8 + tig) : 0u;
            qa[ks][1] = bB >= 0 ? __ldg(qB + ks * 8 + tig) : 0u;
            qa[ks][2] = bA >= 0 ? __ldg(qA + ks * 8 + 4 + tig) : 0u;
            qa[ks][3] = bB >= 0 ? __ldg(qB + ks * 8 + 4 + tig) : 0u;
        }
    }
    float o[C::DT][4];
#pragma unroll
    for (int dt = 0; dt < C::DT; ++dt)
#pragma unroll
        for (int i = 0; i < 4; ++i) o[dt][i] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    const float sl2 = p.scale_log2;
    // lane-dependent parts of the ldmatrix row addresses
    const int kq = lane >> 3, kr = lane & 7;

    Ring ring;
    for (int c = c0; c < c_end; ++c) {
        if (ctrl[0] || !mbar_wait(&full[ring.stage], ring.phase)) {
            if (lane == 0 && !ctrl[0]) {
                ctrl[0] = 1;
                raise_error(p.err, PKV_DEVERR_TIMEOUT);
            }
            return;
        }
        const int ntok = st_ntok[ring.stage];
        const unsigned bad = st_bad[ring.stage];
        const bool whole = ntok == kPrefixCH && bad == 0;
        const uint32_t skb = smem_addr(smem + ring.stage * C::STAGE_BYTES);
        const uint32_t svb = skb + C::KV_BYTES;
        const int tbase = c * kPrefixCH;

        // Two halves of 32 tokens, each a full online-softmax step: fewer
        // live score registers keep two CTAs per SM within the register file.
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            // S = Q . K^T over 4 token tiles of 8; K rows (tokens) as the B operand
            float sc[4][4];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int trow = (hf * 4 + nt) * 8;
#pragma unroll
                for (int i = 0; i < 4; ++i) sc[nt][i] = 0.f;
#pragma unroll
                for (int k2 = 0; k2 < C::KS / 2; ++k2) {
                    uint32_t r[4];
                    ldsm_x4(swz(skb, trow + kr, k2 * 32 + kq * 8, C::HALF_BYTES), r);
                    mma_bf16(sc[nt], qa[2 * k2], r[0], r[1]);
                    mma_bf16(sc[nt], qa[2 * k2 + 1], r[2], r[3]);
                }
            }
            // mask (chunk tail, bad blocks, each row's own length), scale to
            // log2 units, running max per row (the 4 lanes of a quad share a row)
            float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = (hf * 4 + nt) * 8 + 2 * tig + (e & 1);
                    bool ok = whole;
                    if (!whole) {
                        const int jrel = ((tbase + tok) >> p.log2_bs) - (tbase >> p.log2_bs);
                        ok = tok < ntok && !((bad >> jrel) & 1u);
                    }
                    ok = ok && tbase + tok < (e < 2 ? LA : LB);
                    const float v = ok ? sc[nt][e] * sl2 : -INFINITY;
                    sc[nt][e] = v;
                    if (e < 2)
                        mxA = fmaxf(mxA, v);
                    else
                        mxB = fmaxf(mxB, v);
                }
            mxA = fmaxf(mxA, __shfl_xor_sync(FULL_MASK, mxA, 1));
            mxA = fmaxf(mxA, __shfl_xor_sync(FULL_MASK, mxA, 2));
            mxB = fmaxf(mxB, __shfl_xor_sync(FULL_MASK, mxB, 1));
            mxB = fmaxf(mxB, __shfl_xor_sync(FULL_MASK, mxB, 2));
            const float nA = fmaxf(mA, mxA), nB = fmaxf(mB, mxB);
            const float refA = nA == -INFINITY ? 0.f : nA, refB = nB == -INFINITY ? 0.f : nB;
            const float alA = exp2f(mA - refA), alB = exp2f(mB - refB);
            mA = nA;
            mB = nB;
            lA *= alA;
            lB *= alB;
#pragma unroll
            for (int dt = 0; dt < C::DT; ++dt) {
                o[dt][0] *= alA;
                o[dt][1] *= alA;
                o[dt][2] *= alB;
                o[dt][3] *= alB;
            }
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                sc[nt][0] = exp2f(sc[nt][0] - refA);
                sc[nt][1] = exp2f(sc[nt][1] - refA);
                sc[nt][2] = exp2f(sc[nt][2] - refB);
                sc[nt][3] = exp2f(sc[nt][3] - refB);
                lA += sc[nt][0] + sc[nt][1];
                lB += sc[nt][2] + sc[nt][3];
            }

            // O += P . V over 2 k-steps of 16 tokens; P from the S accumulator
            // (token tiles 2kt, 2kt+1 of this half), split into bf16 hi + lo
#pragma unroll
            for (int kt = 0; kt < 2; ++kt) {
                const int t16 = hf * 32 + kt * 16;  // first token of the k-step
                uint32_t ph[4], pl[4];
                {
                    const float* s0 = sc[2 * kt];
                    const float* s1 = sc[2 * kt + 1];
                    ph[0] = pack_bf16(s0[0], s0[1]);
                    ph[1] = pack_bf16(s0[2], s0[3]);
                    ph[2] = pack_bf16(s1[0], s1[1]);
                    ph[3] = pack_bf16(s1[2], s1[3]);
                    pl[0] = pack_bf16(s0[0] - bf16_round(s0[0]), s0[1] - bf16_round(s0[1]));
                    pl[1] = pack_bf16(s0[2] - bf16_round(s0[2]), s0[3] - bf16_round(s0[3]));
                    pl[2] = pack_bf16(s1[0] - bf16_round(s1[0]), s1[1] - bf16_round(s1[1]));
                    pl[3] = pack_bf16(s1[2] - bf16_round(s1[2]), s1[3] - bf16_round(s1[3]));
                }
                // V tokens this lane's B fragments carry: t16 + 2tig (+1), and + 8
                uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
                if (!whole) {
                    auto valid = [&](int tok) {
                        const int jrel = ((tbase + tok) >> p.log2_bs) - (tbase >> p.log2_bs);
                        return tok < ntok && !((bad >> jrel) & 1u);
                    };
                    const int t = t16 + 2 * tig;
                    keep0 = (valid(t) ? 0x0000ffffu : 0u) | (valid(t + 1) ? 0xffff0000u : 0u);
                    keep1 = (valid(t + 8) ? 0x0000ffffu : 0u) | (valid(t + 9) ? 0xffff0000u : 0u);
                }
#pragma unroll
                for (int d2 = 0; d2 < C::DT / 2; ++d2) {
                    uint32_t r[4];
                    ldsm_x4_t(swz(svb, t16 + kr + 8 * (kq & 1), d2 * 16 + 8 * (kq >> 1),
                                  C::HALF_BYTES),
                              r);
                    r[0] &= keep0;
                    r[1] &= keep1;
                    r[2] &= keep0;
                    r[3] &= keep1;
                    mma_bf16(o[2 * d2], ph, r[0], r[1]);
                    mma_bf16(o[2 * d2], pl, r[0], r[1]);
                    mma_bf16(o[2 * d2 + 1], ph, r[2], r[3]);
                    mma_bf16(o[2 * d2 + 1], pl, r[2], r[3]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[ring.stage]);
        ring.advance(kStagesP);
    }

    // the row sums: add the quad's partials
    lA += __shfl_xor_sync(FULL_MASK, lA, 1);
    lA += __shfl_xor_sync(FULL_MASK, lA, 2);
    lB += __shfl_xor_sync(FULL_MASK, lB, 1);
    lB += __shfl_xor_sync(FULL_MASK, lB, 2);
    // partial state of this split for rows A and B
    if (bA >= 0) {
        const size_t row = ((size_t)sp * p.num_seqs + bA) * p.num_q_heads + hA;
        if (tig == 0) {
            p.pfx_ml[row * 2] = mA;
            p.pfx_ml[row * 2 + 1] = lA;
        }
        float* ra = p.pfx_acc + row * D;
#pragma unroll
        for (int dt = 0; dt < C::DT; ++dt)
            *reinterpret_cast<float2*>(ra + dt * 8 + 2 * tig) = make_float2(o[dt][0], o[dt][1]);
    }
    if (bB >= 0) {
        const size_t row = ((size_t)sp * p.num_seqs + bB) * p.num_q_heads + hB;
        if (tig == 0) {
            p.pfx_ml[row * 2] = mB;
            p.pfx_ml[row * 2 + 1] = lB;
        }
        float* ra = p.pfx_acc + row * D;
#pragma unroll
        for (int dt = 0; dt < C::DT; ++dt)
            *reinterpret_cast<float2*>(ra + dt * 8 + 2 * tig) = make_float2(o[dt][2], o[dt][3]);
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
