// decode_mma.cu -- paged decode attention with the q.K^T and P.V contractions
// on the tensor cores (bf16 operands, fp32 accumulation), for bf16 caches with
// block_size >= 8.
//
// What it computes ("PagedAttention: Optimizing KV Cache Utilization in Large
// Language Models", "The Math: Block Attention Calculation", read as one
// softmax over the whole request): for request b and query head h,
//     out[b,h,:] = sum_t softmax_t(scale * q[b,h,:] . K_t) V_t,
// with K_t / V_t located through the request's block table ("The Mechanics of
// PagedAttention").
//
// Why tensor cores on an HBM-bound path: the CUDA-core version executes ~0.17
// instructions per DRAM byte, which would need ~97 % of the SM issue ceiling at
// the HBM copy peak.  Here a 16-token tile costs ~50 warp instructions.
//
// Shapes per 16-token tile (tokens are the MMA M dimension, the query heads of
// the group -- padded to 8 per n-tile -- are N, so one K/V read serves the whole
// group):
//   S^T[16 x 8]  = K[16 x d] . Q^T[d x 8]        (d/16 mma.m16n8k16, A = K via ldmatrix)
//   O^T[d x 8]  += V^T[d x 16] . P^T[16 x 8]     (d/16 mma per split, A = V^T via ldmatrix.trans)
// P^T comes from the S^T accumulator: exp2 in fp32, packed to bf16 and moved
// into the B-operand layout with movmatrix.trans.  P is split into bf16 hi + lo
// parts (two MMAs) so the weights keep ~16 mantissa bits.
//
// Data movement: producer warps walk the block table (32 entries per
// coalesced load, next window prefetched, next segment's first window too) and
// issue TMA tensor copies (2-D or 3-D tensor map over the cache rows, 128-byte
// swizzle, no multicast) of each physical block's K and V rows into a ring of
// shared-memory stages with mbarrier completion, one lane per block.
// Consumer warps do the math, taking the CTA's 64-token chunks in turn, and
// hand their running state to an epilogue warp: bf16 one CTA per SM with one
// producer and two consumers (16-head groups: one consumer, two CTAs per SM);
// fp8 one CTA per SM with four producers and six consumers that widen the
// codes to f16 in registers.  The epilogue normalises; a (request, head group)
// split over several units is merged in-kernel by the last unit to finish
// (per-group arrival counter and ready flags in the workspace, reset by the
// merger), or -- fixed partitions and prefix groups -- by a separate merge
// kernel:
//   out = sum_u 2^(m_u - M) acc_u / sum_u 2^(m_u - M) l_u.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include <algorithm>
#include <mutex>

#include "decode_common.cuh"
#include "mma_ptx.cuh"

namespace pkv {
namespace {

constexpr int kCH = 64;         // tokens per stage
constexpr int kMT = kCH / 16;   // 16-token MMA tiles per stage
constexpr int kRingBudget = 104448;  // 3 stages of K+V+q at head_dim 128

constexpr int cmin(int a, int b) { return a < b ? a : b; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int cgcd(int a, int b) { return b == 0 ? a : cgcd(b, a % b); }
constexpr int clcm(int a, int b) { return a / cgcd(a, b) * b; }

// F8 = false: bf16 cache, tiles land swizzled and feed bf16 MMAs directly.
// F8 = true : fp8 (e4m3) cache, tiles land as rows of head_dim one-byte codes
//             (TMA boxes with the swizzle of their width) and every consumer
//             widens what it loads from them to f16 in registers (exact), for
//             f16 MMAs; q is widened to f16 likewise.
template <int D, int NT, bool F8, bool SOLO = false, bool RC = false>
struct MmaCfg {
    static constexpr int NHALF = D / 64;            // 128-byte column halves of a 16-bit row
    static constexpr int KS = D / 16;               // k-steps of q.K^T, m-tiles of P.V
    static constexpr int HALF_BYTES = kCH * 128;    // one swizzled half region (16-bit data)
    static constexpr int KV_BYTES = F8 ? kCH * D : NHALF * HALF_BYTES;  // K (or V) of a stage
    static constexpr int GP = 8 * NT;               // query heads per head group (padded)
    static constexpr int Q_BYTES = GP * D * 2;      // the group's q rows (first stage of a segment)
    // Consumers.  bf16, 16-head groups: one tensor-core consumer reads every
    // stage (two CTAs per SM).  Otherwise one CTA per SM whose NCONS consumers
    // take the CTA's chunks in turn (chunk n -> consumer n % NCONS, stage
    // n % NSTAGE; NSTAGE is a multiple of NCONS, so a stage always serves the
    // same consumer and each barrier has one waiter stepping through its
    // phases in order):
    //   bf16, 8-head groups, TMA boxes: two consumers.  One CTA per SM halves the units
    //     of a call, so a unit (56 chunks of the 4k batch) is nearly as long
    //     as a (request, kv head) group (64): most groups split into two
    //     parts, one of which finishes early and is prefetched by the other's
    //     merge -- with two CTAs per SM a group's middle parts end with the
    //     kernel and the last merges wait for them.  SOLO keeps two CTAs
    //     per SM with one consumer each, for calls of many (request, head
    //     group) pairs, where few groups split and two epilogue warps per SM
    //     share the many short segments.
    //   bf16, 8-head groups, row copies (blocks of 2 or 4 rows): three
    //     consumers -- each tile's rows come from several blocks (per-row
    //     addresses) and q from global memory, work two consumers left
    //     exposed (block size 4: 60.1 -> 53.3 us back to back); the TMA
    //     path is better with two.
    //   fp8: widening codes costs instructions and latency the bf16 path does
    //     not have, and one consumer warp cannot hide its own ldmatrix -> cvt
    //     -> mma chains: six consumers (two on each of two SM sub-partitions)
    //     overlap them; the 16-head configuration keeps four (its consumers
    //     need all the registers).
    static constexpr int NCONS = F8 ? (NT == 1 ? 6 : 4) : (NT == 1 && !SOLO ? (RC ? 3 : 2) : 1);
    // bf16: K | V | q, rounded to the 1 KB the 128-byte swizzle pattern
    // repeats on, or the row-copy regions if larger; the first NCONS stages
    // of a segment -- each consumer's first chunk of it -- carry the group's q
    // (row copies: the consumer reads it from global memory).  fp8: K | V only
    // (8 or 4 KB each, whole swizzle periods); each consumer reads the group's
    // q from global memory.
    static constexpr bool Q_IN_STAGE = !F8;
    // row-copy stages (bf16 blocks of 2 or 4 rows): K | V regions of up to 32
    // skewed blocks (rc_block_bytes), inside the same stage size
    static constexpr int RC_KV_BYTES = kCH * D * 2 + 32 * 16;
    static constexpr int STAGE_BYTES =
        F8 ? 2 * KV_BYTES
           : (cmax(2 * KV_BYTES + (Q_IN_STAGE ? Q_BYTES : 0), 2 * RC_KV_BYTES) + 1023) / 1024 * 1024;
    static_assert(F8 || 2 * RC_KV_BYTES <= STAGE_BYTES, "row-copy regions fit a stage");
    // producer warps: a TMA issue holds the issuing warp ~0.11 us, so one
    // warp issues at most ~9 boxes per us however its lanes share them.  An
    // fp8 chunk is 8 boxes of 2 KB; four producers take chunks in turn (stage
    // n % NSTAGE belongs to producer n % NPROD), enough to keep 12 stages in
    // flight.  The 16-head configuration keeps two (registers).  bf16 with one
    // CTA per SM: two (a chunk of 8-row blocks is 16 boxes), three for row
    // copies (32 or 64 bulk copies per chunk); two CTAs: one each.
    static constexpr int NPROD = F8 ? (NT == 1 ? 4 : 2) : (NCONS > 1 ? (RC ? 3 : 2) : 1);
    static constexpr int THREADS = 32 * (NPROD + NCONS + 1);  // + the epilogue
    // consumer -> epilogue hand-off: per lane, the accumulators and (m, l);
    // NDUMP slots per consumer (two, so a consumer can hand over a short
    // segment while the epilogue still merges the previous one, where the
    // shared memory allows)
    static constexpr int DUMP_BYTES = (KS * NT * 4 + NT * 4) * 32 * 4;
    static constexpr int NDUMP = NCONS <= 2 ? 2 : 1;
    // One CTA per SM: as many stages as the shared memory holds beside the
    // hand-off slots (up to 24), a multiple of NCONS and NPROD: 192 KB or
    // more in flight per SM at head_dim 128.
    static constexpr int RING = 227 * 1024 - NCONS * NDUMP * DUMP_BYTES - 4096;
    static constexpr int STAGE_STEP = clcm(NCONS, NPROD);
    static constexpr int NSTAGE = NCONS == 1 ? cmax(2, cmin(8, kRingBudget / STAGE_BYTES))
                                             : cmin(24, RING / STAGE_BYTES) / STAGE_STEP * STAGE_STEP;
    static_assert(NSTAGE % NPROD == 0 && NSTAGE % NCONS == 0 && NSTAGE >= 2,
                  "each stage belongs to one producer and one consumer");
};

// ---- shared-memory layout ------------------------------------------------------

template <int D, int NT, bool F8, bool SOLO = false, bool RC = false>
struct Smem {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    // consumer -> epilogue hand-off slots per consumer
    static constexpr int NDUMP = C::NDUMP;
    static constexpr int NSLOT = C::NCONS * NDUMP;
    static constexpr int DUMP_ACC = C::KS * NT * 4;       // acc registers per lane
    static constexpr int DUMP_ML = NT * 4;                // m[2], l[2] per n-tile per lane
    static constexpr int DUMP_BYTES = C::DUMP_BYTES;
    static constexpr int OFF_DUMP = C::NSTAGE * C::STAGE_BYTES;
    // fp8, 8-head groups: one partial record (acc rows, then m/l pairs) the
    // epilogue prefetches for a split group's merge
    static constexpr int PF_BYTES = (F8 && NT == 1) ? C::GP * D * 4 + C::GP * 2 * 4 : 0;
    static constexpr int OFF_PF = OFF_DUMP + NSLOT * DUMP_BYTES;
    static constexpr int OFF_BAR = OFF_PF + PF_BYTES;
    // full/empty per stage, dfull/dempty per dump slot
    static constexpr int OFF_META = OFF_BAR + (2 * C::NSTAGE + 2 * NSLOT) * 8;
    // ntok/bad per stage
    static constexpr int OFF_CTRL = OFF_META + 2 * C::NSTAGE * 4;
    static constexpr int BYTES = OFF_CTRL + 16 + 1024;   // + alignment slack
    static_assert(BYTES <= 227 * 1024, "within the opt-in shared memory of one CTA");
};

// Head-dim index of accumulator element (dt, lane group grp, upper half hi) of
// P.V.  bf16: the natural m16n8 rows, 16 dt + grp + 8 hi.  fp8: the consumer
// loads V with ldmatrix on byte pairs, so lane group grp of m-tile dt holds
// dims 16 dt + 4 (grp / 2) + grp % 2 (+ 2 for the upper half).
template <bool F8>
__device__ __forceinline__ int dcol(int dt, int grp, int hi) {
    if constexpr (F8)
        return dt * 16 + 4 * (grp >> 1) + (grp & 1) + 2 * hi;
    else
        return dt * 16 + grp + 8 * hi;
}

// fp8 stage rows are D bytes landed by TMA with the swizzle of their width:
// 16-byte chunk c of row r sits at chunk c ^ f8_swz(r) (128-byte rows: r mod 8;
// 64-byte rows: (r / 2) mod 4).  Stage regions start on the pattern's period.
template <int D>
__device__ __forceinline__ int f8_swz(int row) {
    if constexpr (D == 128)
        return row & 7;
    else
        return (row >> 1) & 3;
}

// Row-copy stages (bf16, blocks of 2 or 4 rows): block j of the chunk holds
// its rows contiguously at j * rc_block_bytes, one 16-byte bank group further
// than a dense packing would put it, so rows of eight consecutive blocks fall
// in eight distinct bank groups.  K and V regions of 32 blocks of 2 rows (the
// larger case) fit inside a bf16 stage.
template <int D>
__device__ __forceinline__ int rc_block_bytes(int block_size) {
    return block_size * D * 2 + 16;
}

// Token (within the 64-token chunk) behind MMA row i of token tile mt in
// row-copy stages: a tile is one in-block row (mt % block_size) of 16
// consecutive blocks, so each 8-row ldmatrix tile reads eight different
// blocks.  q.K^T and P.V use the same mapping, so the token order inside the
// chunk is immaterial.
__device__ __forceinline__ int rc_token(int mt, int i, int log2_bs) {
    const int bs = 1 << log2_bs;
    return bs * (16 * (mt >> log2_bs) + i) + (mt & (bs - 1));
}

// bf16 stages hold each block's rows as one TMA box of [half][rb rows][128 B]
// (rb = min(block_size, 64), both 64-column halves of a 128-dim row in one
// box), blocks one after another: byte offset of 64-column half `half` of
// stage row t (t < 64).  The 128-byte swizzle is keyed on t % 8, since every
// box starts on a 1 KB boundary.
template <int NHALF>
__device__ __forceinline__ int bf16_row_off(int t, int half, int log2_rb) {
    const int rb = 1 << log2_rb;
    return (t >> log2_rb) * (rb * NHALF * 128) + half * (rb * 128) + (t & (rb - 1)) * 128;
}

// ---- producer ------------------------------------------------------------------

// RC: blocks of 2 or 4 rows (bf16), copied row by row instead of by TMA boxes;
// a separate instance so the boxed producer carries no trace of it.  APP: the
// fused append (bf16, one CTA per SM), likewise a separate instance: a plain
// decode's chunk loop carries no trace of it.
template <int D, int NT, bool F8, bool RC, bool SOLO, bool APP>
struct Producer {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    static_assert(!(RC && F8), "row copies serve bf16 caches only");
    static_assert(!(APP && F8), "the fused append serves bf16 caches only");

    const DecodeParams& p;
    const CUtensorMap* tmk;
    const CUtensorMap* tmv;
    unsigned char* smem;
    uint64_t* full;
    uint64_t* empty;
    int* st_ntok;
    unsigned* st_bad;
    volatile int* ctrl;
    int lane;
    uint64_t policy;
    int me = 0;              // this producer (chunks n with n % NPROD == me)
    unsigned n_chunk = 0;    // chunks of the CTA so far (all producers')
    unsigned last_n = 0;     // the last chunk this producer issued
    int issued = 0;
    bool waited = false;

    __device__ int load_window(const Cursor& cur, int wbase) const {
        const int nblk = (cur.L + p.block_size - 1) >> p.log2_bs;
        const int j = wbase + lane;
        return j < nblk ? __ldg(p.block_tables + (size_t)cur.b * p.max_blocks + j) : -1;
    }

    static __device__ __forceinline__ int first_block(const Cursor& cur, int c0, int log2_bs) {
        return (cur.t0 + c0 * kCH) >> log2_bs;
    }

    // Fused append.  The new token of request cur.b (its last, position
    // L - 1): this lane's 16-byte vector of its K (lanes 0 ..) or V (lanes
    // 16 ..) row of kv head kvh, loaded when the segment that holds it starts,
    // so the load is in flight while the segment's earlier chunks are issued.
    static constexpr int kAppVec = D * 2 / 16;  // 16-byte vectors per row
    __device__ __forceinline__ uint4 append_load(int b, int kvh) const {
        const size_t src = ((size_t)b * p.num_kv_heads + kvh) * D;
        const uint4* from = reinterpret_cast<const uint4*>(
            static_cast<const __nv_bfloat16*>(lane < 16 ? p.k_new : p.v_new) + src);
        return (lane & 15) < kAppVec ? __ldg(from + (lane & 15)) : make_uint4(0u, 0u, 0u, 0u);
    }
    // ... then stored to its slot just before the copies of the chunk that
    // holds it are issued; the proxy fence orders these generic writes before
    // the copy engine's reads of the block.
    __device__ __forceinline__ void append_store(const Cursor& cur, int kvh, int tab, int wbase,
                                                 uint4 row) {
        const int t = cur.L - 1;
        const int phys = __shfl_sync(FULL_MASK, tab, (t >> p.log2_bs) - wbase);
        if (phys >= 0 && phys < p.num_blocks && (lane & 15) < kAppVec) {
            const size_t dst = ((size_t)phys * p.num_kv_heads + kvh) * p.block_size * D +
                               (size_t)(t & (p.block_size - 1)) * D;
            uint4* to = reinterpret_cast<uint4*>(
                static_cast<__nv_bfloat16*>(const_cast<void*>(lane < 16 ? p.k_cache : p.v_cache)) +
                dst);
            to[lane & 15] = row;
            fence_proxy_async_global();
        }
        __syncwarp();
    }

    // Returns false when the CTA must stop (a wait gave up).
    __device__ bool run_segment(const Segment& sg, int tab_first) {
        const Cursor& cur = sg.cur;
        const int kvh = cur.hg / p.num_sub, sub = cur.hg % p.num_sub;
        const int hq0 = kvh * p.group + sub * C::GP;
        const int gv = min(C::GP, p.group - sub * C::GP);
        const int nblk = (cur.L + p.block_size - 1) >> p.log2_bs;
        const int rb = min(p.block_size, kCH);  // rows per TMA box
        // Table windows start at the segment's first block and advance by 32
        // blocks, a whole number of chunks (64 / block_size blocks each), so
        // no chunk straddles two windows whatever block the request's pass
        // starts at.
        int wbase = first_block(cur, sg.c0, p.log2_bs);
        int tab = tab_first;
        int tab_next = (wbase + 32 < nblk) ? load_window(cur, wbase + 32) : -1;
        uint4 app_row = make_uint4(0u, 0u, 0u, 0u);
        if constexpr (APP) {
            if (!waited) {
                griddep_wait();  // the new rows may come from the previous kernel
                waited = true;
            }
            // this producer issues the group's last chunk (the new token's)
            const unsigned n_last = n_chunk + (unsigned)(sg.c1 - 1 - sg.c0);
            if (sg.c1 == cur.nch && (C::NPROD == 1 || (int)(n_last % C::NPROD) == me))
                app_row = append_load(cur.b, kvh);
        }
        for (int c = sg.c0; c < sg.c1; ++c) {
            const int t0 = cur.t0 + c * kCH;
            const int ntok = min(kCH, cur.L - t0);
            const int ja = t0 >> p.log2_bs;
            const int jb = (t0 + ntok - 1) >> p.log2_bs;
            if (ja >= wbase + 32) {
                wbase += 32;
                tab = tab_next;
                tab_next = (wbase + 32 < nblk) ? load_window(cur, wbase + 32) : -1;
            }
            const unsigned n = n_chunk++;
            if (C::NPROD > 1 && (int)(n % C::NPROD) != me) continue;  // the other producer's
            const int stage = (int)(n % C::NSTAGE);
            const uint32_t phase = (n / C::NSTAGE) & 1u;
            int ok = 1;
            if (lane == 0) ok = !ctrl[0] && mbar_wait(&empty[stage], phase ^ 1u, p.wait_ns);
            ok = __shfl_sync(FULL_MASK, ok, 0);
            if (!ok) {
                if (lane == 0) {
                    ctrl[0] = 1;
                    raise_error(p.err, PKV_DEVERR_TIMEOUT);
                }
                return false;
            }
            if (!waited) {
                // K/V and q may come from the previous kernel in the stream.
                griddep_wait();
                waited = true;
            }
            if (p.fault_mode == kFaultSkipStage && blockIdx.x == 0 && (int)n == p.fault_arg) {
                // test-only fault: this stage is never filled, so its
                // consumer's bounded wait runs out (nothing is in flight)
                ++issued;
                last_n = n;
                continue;
            }
            uint32_t nvalid = 0, bad = 0;
            for (int j = ja; j <= jb; ++j) {
                const int phys = __shfl_sync(FULL_MASK, tab, j - wbase);
                if (phys < 0 || phys >= p.num_blocks)
                    bad |= 1u << (j - ja);
                else
                    ++nvalid;
            }
            if constexpr (APP) {
                if (c == cur.nch - 1) append_store(cur, kvh, tab, wbase, app_row);
            }
            unsigned char* sk = smem + stage * C::STAGE_BYTES;
            unsigned char* sv = sk + C::KV_BYTES;
            unsigned char* sq = sv + C::KV_BYTES;
            if constexpr (RC) {
                // Blocks of 2 or 4 rows: a block's rows of one kv head are one
                // contiguous run of block_size * D bf16, fetched with one bulk
                // copy per (block, K or V) -- 32 or 64 per chunk, one or two
                // per lane -- into the skewed layout of rc_block_bytes().  The
                // consumer reads q from global memory.
                const uint32_t run = (uint32_t)p.block_size * D * 2u;
                if (lane == 0) {
                    st_ntok[stage] = ntok;
                    st_bad[stage] = bad;
                    if (bad) raise_error(p.err, PKV_DEVERR_BAD_BLOCK);
                    mbar_arrive_expect_tx(&full[stage], nvalid * 2u * run);
                }
                __syncwarp();  // the expect-tx above comes first
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int cp = lane + 32 * it;  // copy cp: block cp / 2, K (even) or V
                    const int jrel = cp >> 1;
                    const int phys = __shfl_sync(FULL_MASK, tab, min(ja + jrel, jb) - wbase);
                    if (ja + jrel <= jb && phys >= 0 && phys < p.num_blocks) {
                        const size_t goff =
                            ((size_t)phys * p.num_kv_heads + kvh) * p.block_size * D * 2;
                        const unsigned char* src =
                            static_cast<const unsigned char*>((cp & 1) ? p.v_cache : p.k_cache) + goff;
                        bulk_load(sk + ((cp & 1) ? C::RC_KV_BYTES : 0) +
                                      jrel * rc_block_bytes<D>(p.block_size),
                                  src, run, &full[stage], policy);
                    }
                }
                ++issued;
                last_n = n;
                continue;
            }
            if (lane == 0) {
                st_ntok[stage] = ntok;
                st_bad[stage] = bad;
                if (bad) raise_error(p.err, PKV_DEVERR_BAD_BLOCK);
                // each consumer's first chunk of the segment carries q
                const uint32_t qbytes =
                    (C::Q_IN_STAGE && c - sg.c0 < C::NCONS) ? (uint32_t)gv * D * 2u : 0u;
                const uint32_t row_bytes = F8 ? (uint32_t)D : (uint32_t)C::NHALF * 128u;
                mbar_arrive_expect_tx(&full[stage], nvalid * 2u * rb * row_bytes + qbytes);
                if (qbytes)  // the group's q rows ride with the stage
                    bulk_load(sq, static_cast<const __nv_bfloat16*>(p.q) +
                                      ((size_t)cur.b * p.num_q_heads + hq0) * D,
                              qbytes, &full[stage], policy);
            }
            // One lane per block of the chunk issues that block's copies: a TMA
            // issue costs the issuing thread ~0.1 us, so lane-parallel issue
            // keeps the copies of a chunk from queueing behind each other.
            __syncwarp();  // the expect-tx above comes first
            {
                const int j = ja + lane;
                const int phys = __shfl_sync(FULL_MASK, tab, min(j, jb) - wbase);
                if (j <= jb && phys >= 0 && phys < p.num_blocks) {
                    // rows of this block in the stage, and where they start in the cache
                    const int srow = (j << p.log2_bs) - t0 > 0 ? (j << p.log2_bs) - t0 : 0;
                    const int boff = t0 - (j << p.log2_bs) > 0 ? t0 - (j << p.log2_bs) : 0;
                    const int grow = (phys * p.num_kv_heads + kvh) * p.block_size + boff;
                    if constexpr (F8) {
                        // whole code rows (D bytes) with the swizzle of their
                        // width, so the consumers' ldmatrix reads are free of
                        // bank conflicts
                        tma_load_2d(sk + srow * D, tmk, 0, grow, &full[stage], policy);
                        tma_load_2d(sv + srow * D, tmv, 0, grow, &full[stage], policy);
                    } else if constexpr (C::NHALF == 2) {
                        // one 3-D box per block holds both 64-column halves of
                        // its rb rows ([half][row][128 B]): half the TMA issues
                        tma_load_3d(sk + srow * 256, tmk, 0, grow, 0, &full[stage], policy);
                        tma_load_3d(sv + srow * 256, tmv, 0, grow, 0, &full[stage], policy);
                    } else {
                        tma_load_2d(sk + srow * 128, tmk, 0, grow, &full[stage], policy);
                        tma_load_2d(sv + srow * 128, tmv, 0, grow, &full[stage], policy);
                    }
                }
            }
            ++issued;
            last_n = n;
        }
        return true;
    }

    // spec_b / spec_j / spec_tab: a table window of request spec_b starting
    // at block spec_j, loaded before the plan was known (spec_b < 0: none);
    // used if the CTA's first segment starts there.
    __device__ void run(SegIter<kCH>& it, int spec_b, int spec_j, int spec_tab) {
        int tab_first = -1;
        if (it.valid) {
            const Segment sg = it.current();
            const int j0 = first_block(sg.cur, sg.c0, p.log2_bs);
            if (sg.cur.b == spec_b && j0 == spec_j) {
                const int nblk = (sg.cur.L + p.block_size - 1) >> p.log2_bs;
                tab_first = j0 + lane < nblk ? spec_tab : -1;
            } else {
                tab_first = load_window(sg.cur, j0);
            }
        }
        while (it.valid) {
            const Segment sg = it.current();
            it.advance(p, lane);
            // prefetch the next segment's first table window before streaming this one
            int tab_after = -1;
            if (it.valid) {
                const Segment nx = it.current();
                tab_after = load_window(nx.cur, first_block(nx.cur, nx.c0, p.log2_bs));
            }
            if (!run_segment(sg, tab_first)) break;
            tab_first = tab_after;
        }
        if (ctrl[0] && lane == 0) {
            // A wait gave up somewhere in the CTA: before this warp exits, wait
            // (bounded) for the stages it issued last, so no copy lands in
            // shared memory after the CTA has gone.
            const int k_max = min(issued, C::NSTAGE / C::NPROD);
            for (int k = 0; k < k_max; ++k) {
                const unsigned nn = last_n - (unsigned)(k * C::NPROD);
                mbar_wait(&full[nn % C::NSTAGE], (nn / C::NSTAGE) & 1u, p.wait_ns);
            }
        }
    }
};

// Per-segment facts every role derives the same way.
struct SegInfo {
    long long u, u_first, u_last;  // the group's units u_first .. u_last
    int nseg;                      // parts of the group (units)
    int hq0, gv, b, kvh;
    size_t bg;
};

template <int GP>
__device__ __forceinline__ SegInfo seg_info(const DecodeParams& p, const Segment& sg, long long W) {
    SegInfo si;
    si.u = sg.u;
    si.u_first = sg.gstart / W;
    si.u_last = (sg.gstart + sg.cur.nch - 1) / W;
    si.nseg = (int)(si.u_last - si.u_first + 1);
    const int kvh = sg.cur.hg / p.num_sub, sub = sg.cur.hg % p.num_sub;
    si.hq0 = kvh * p.group + sub * GP;
    si.gv = min(GP, p.group - sub * GP);
    si.b = sg.cur.b;
    si.kvh = kvh;
    si.bg = (size_t)sg.cur.b * p.num_hg + sg.cur.hg;
    return si;
}

// ---- consumer (tensor-core math) ----------------------------------------------

// Consumer `me` (0 .. NCONS-1): takes the CTA's chunks n with n % NCONS == me
// (stage n % NSTAGE).  bf16: K and V as 16-bit swizzled tiles; the group's q
// from the segment's first stage (one consumer) or from global memory.  fp8:
// widens the e4m3 codes in registers: ldmatrix on byte pairs gives lane
// (grp, tig) four consecutive codes of one token row, which one cvt per pair
// turns into two f16x2 words.
//   q.K^T: the four codes 4 tig .. 4 tig + 3 of a 16-code block serve as the A
//     fragment's k = 2 tig, 2 tig + 1 and 2 tig + 8, 2 tig + 9, a fixed
//     permutation of the head dim inside each block; q is loaded with the same
//     permutation (dims 4 tig .. 4 tig + 3), so the dot products are unchanged.
//   P.V: the widened words are 8 x 8 tiles with tokens as rows; movmatrix.trans
//     makes them A fragments of V^T with tokens as k, and the head-dim rows
//     come out permuted as dcol<true> describes.
template <int D, int NT, bool F8, bool RC, bool SOLO>
__device__ __forceinline__ void consume(const DecodeParams& p, SegIter<kCH>& it,
                                        unsigned char* smem, uint64_t* full, uint64_t* empty,
                                        uint64_t* dfull, uint64_t* dempty, const int* st_ntok,
                                        const unsigned* st_bad, volatile int* ctrl, int lane,
                                        int me) {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    using S = Smem<D, NT, F8, SOLO, RC>;
    constexpr int GP = C::GP;
    const int grp = lane >> 2, tig = lane & 3;
    const int mi = lane >> 3, r8 = lane & 7;
    // ldmatrix row/chunk components that depend only on the lane
    const int k_row = r8 + 8 * (mi & 1), k_cx = mi >> 1;  // K (A operand); fp8: K and V
    const int v_row = r8 + 8 * (mi >> 1), v_cx = mi & 1;  // bf16 V^T (transposed load)
    Ring ring, dring;
    unsigned n_chunk = 0;  // several consumers: chunks of the CTA so far
    bool waited = false;   // q read from global memory: after the grid dependency
    // bf16 stages: byte offsets of this lane's ldmatrix rows per token tile
    const int log2_rb = min(p.log2_bs, 6);
    int k_off[kMT], v_off[kMT];
#pragma unroll
    for (int mt = 0; mt < kMT; ++mt) {
        k_off[mt] = bf16_row_off<C::NHALF>(mt * 16 + k_row, 0, log2_rb);
        v_off[mt] = bf16_row_off<C::NHALF>(mt * 16 + v_row, 0, log2_rb);
    }

    while (it.valid) {
        const Segment sg = it.current();
        it.advance(p, lane);
        const SegInfo si = seg_info<GP>(p, sg, it.W);
        // softmax scale in log2 units, times the K dequantisation scale for fp8
        const float s_log2 = F8 ? p.scale_log2 * __ldg(p.k_scale + si.kvh) : p.scale_log2;

        uint32_t qb[NT][C::KS][2];
        float m[NT][2], l[NT][2], acc[C::KS][NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
            for (int dt = 0; dt < C::KS; ++dt)
#pragma unroll
                for (int i = 0; i < 4; ++i) acc[dt][nt][i] = 0.f;
        }

        bool have_q = false;
        if constexpr (!C::Q_IN_STAGE || RC) {
            // Q^T B-fragments straight from global memory, head nt*8+grp.
            // fp8: the permuted order, dims 16 ks + 4 tig, +1 (b0) and
            // 16 ks + 4 tig + 2, +3 (b1), widened bf16 -> f16.  bf16: the
            // natural order, dims 16 ks + 2 tig, +1 (b0) and + 8, + 9 (b1).
            // Only a consumer with a chunk of this segment needs them.
            bool any = C::NCONS == 1;
            if constexpr (C::NCONS > 1)
                for (unsigned n = n_chunk; n < n_chunk + (unsigned)(sg.c1 - sg.c0); ++n)
                    any |= (int)(n % C::NCONS) == me;
            if (any) {
                if (!waited) {
                    griddep_wait();  // q may come from the previous kernel
                    waited = true;
                }
                const __nv_bfloat16* gq =
                    static_cast<const __nv_bfloat16*>(p.q) + ((size_t)si.b * p.num_q_heads + si.hq0) * D;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + grp;
#pragma unroll
                    for (int ks = 0; ks < C::KS; ++ks) {
                        if constexpr (F8) {
                            uint2 w = make_uint2(0u, 0u);
                            if (h < si.gv)
                                w = __ldg(reinterpret_cast<const uint2*>(gq + (size_t)h * D + ks * 16 + 4 * tig));
                            qb[nt][ks][0] = bf16x2_to_f16x2(w.x);
                            qb[nt][ks][1] = bf16x2_to_f16x2(w.y);
                        } else {
                            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(gq + (size_t)h * D);
                            qb[nt][ks][0] = h < si.gv ? __ldg(q32 + ks * 8 + tig) : 0u;
                            qb[nt][ks][1] = h < si.gv ? __ldg(q32 + ks * 8 + 4 + tig) : 0u;
                        }
                    }
                }
                have_q = true;
            }
        }

        for (int c = sg.c0; c < sg.c1; ++c) {
            int stage;
            uint32_t phase;
            if constexpr (C::NCONS > 1) {
                const unsigned n = n_chunk++;
                if ((int)(n % C::NCONS) != me) continue;
                stage = (int)(n % C::NSTAGE);
                phase = (n / C::NSTAGE) & 1u;
            } else {
                stage = ring.stage;
                phase = ring.phase;
            }
            if (ctrl[0] || !mbar_wait(&full[stage], phase, p.wait_ns)) {
                if (lane == 0 && !ctrl[0]) {
                    ctrl[0] = 1;
                    raise_error(p.err, PKV_DEVERR_TIMEOUT);
                }
                return;
            }
            const int ntok = st_ntok[stage];
            const unsigned bad = st_bad[stage];
            unsigned char* sk = smem + stage * C::STAGE_BYTES;
            unsigned char* sv = sk + (RC ? C::RC_KV_BYTES : C::KV_BYTES);
            const bool whole = ntok == kCH && bad == 0;

            if (C::Q_IN_STAGE && !RC && !have_q) {
                // This consumer's first chunk of the segment carries the group's q.
                // Q^T B-fragments: head nt*8+grp, dims ks*16 + 2*tig (+1) and +8 (+9).
                have_q = true;
                const uint32_t* sq = reinterpret_cast<const uint32_t*>(sv + C::KV_BYTES);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int h = nt * 8 + grp;
#pragma unroll
                    for (int ks = 0; ks < C::KS; ++ks) {
                        qb[nt][ks][0] = h < si.gv ? sq[h * (D / 2) + ks * 8 + tig] : 0u;
                        qb[nt][ks][1] = h < si.gv ? sq[h * (D / 2) + ks * 8 + 4 + tig] : 0u;
                    }
                }
            }

            const uint32_t skb = smem_addr(sk), svb = smem_addr(sv);

            if (!F8 && !RC && !whole) {
                // Rows of tokens that do not take part (past the end, or in a
                // block the table got wrong) may hold stale or poisoned data:
                // zero their V rows so 0-weight x NaN cannot reach the sum.
                for (int idx = lane; idx < kCH * C::NHALF * 8; idx += 32) {
                    const int row = idx / (C::NHALF * 8);
                    const int rest = idx % (C::NHALF * 8);
                    const int jrel = ((c * kCH + row) >> p.log2_bs) - ((c * kCH) >> p.log2_bs);
                    const bool valid = row < ntok && !((bad >> jrel) & 1u);
                    if (!valid)
                        *reinterpret_cast<uint4*>(sv + bf16_row_off<C::NHALF>(row, rest >> 3, log2_rb) +
                                                  (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
                }
                __syncwarp();
            }

            // ---- S^T = K . Q^T for the stage's 4 token tiles ----
            float s[kMT][NT][4];
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) s[mt][nt][i] = 0.f;
            if constexpr (F8) {
                // one ldmatrix.x4 = 16 token rows x 32 codes = two k-steps
#pragma unroll
                for (int j = 0; j < C::KS / 2; ++j) {
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        const int row = mt * 16 + k_row;
                        uint32_t r[4];
                        ldsm_x4(skb + row * D + (((2 * j + k_cx) ^ f8_swz<D>(row)) << 4), r);
                        uint32_t a[2][4];
                        e4m3x4_to_f16(r[0], a[0][0], a[0][2]);
                        e4m3x4_to_f16(r[1], a[0][1], a[0][3]);
                        e4m3x4_to_f16(r[2], a[1][0], a[1][2]);
                        e4m3x4_to_f16(r[3], a[1][1], a[1][3]);
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt)
                                mma_f16(s[mt][nt], a[h], qb[nt][2 * j + h][0], qb[nt][2 * j + h][1]);
                    }
                }
            } else if constexpr (RC) {
                // rows of tile mt: token rc_token(mt, row), unswizzled in its block
#pragma unroll
                for (int mt = 0; mt < kMT; ++mt) {
                    const int tok = rc_token(mt, k_row, p.log2_bs);
                    const uint32_t rb = skb + (tok >> p.log2_bs) * rc_block_bytes<D>(p.block_size) +
                                        (tok & (p.block_size - 1)) * D * 2;
#pragma unroll
                    for (int ks = 0; ks < C::KS; ++ks) {
                        uint32_t a[4];
                        ldsm_x4(rb + ((2 * ks + k_cx) << 4), a);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_bf16(s[mt][nt], a, qb[nt][ks][0], qb[nt][ks][1]);
                    }
                }
            } else {
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks) {
                    const int half = ks >> 2;
                    const int chunk = (2 * (ks & 3) + k_cx) ^ r8;
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        uint32_t a[4];
                        ldsm_x4(skb + k_off[mt] + half * (128 << log2_rb) + (chunk << 4), a);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) mma_bf16(s[mt][nt], a, qb[nt][ks][0], qb[nt][ks][1]);
                    }
                }
            }

            // ---- scale, mask, online softmax (base 2) ----
            bool grew = false;
            float alpha[NT][2];
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) s[mt][nt][i] *= s_log2;
                if (!whole) {
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int row = RC ? rc_token(mt, grp + 8 * hi, p.log2_bs) : mt * 16 + grp + 8 * hi;
                        const int jrel = ((c * kCH + row) >> p.log2_bs) - ((c * kCH) >> p.log2_bs);
                        const bool valid = row < ntok && !((bad >> jrel) & 1u);
                        if (!valid) {
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                s[mt][nt][2 * hi] = -INFINITY;
                                s[mt][nt][2 * hi + 1] = -INFINITY;
                            }
                        }
                    }
                }
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float mx = fmaxf(s[0][nt][j], s[0][nt][j + 2]);
#pragma unroll
                    for (int mt = 1; mt < kMT; ++mt) mx = fmaxf(mx, fmaxf(s[mt][nt][j], s[mt][nt][j + 2]));
                    mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(FULL_MASK, mx, 16));
                    const float mnew = fmaxf(m[nt][j], mx);
                    const float mref = mnew == -INFINITY ? 0.f : mnew;
                    grew |= mnew > m[nt][j];
                    alpha[nt][j] = exp2f(m[nt][j] - mref);
                    m[nt][j] = mnew;
                    float ps = 0.f;
#pragma unroll
                    for (int mt = 0; mt < kMT; ++mt) {
                        s[mt][nt][j] = ex2_ftz(s[mt][nt][j] - mref);
                        s[mt][nt][j + 2] = ex2_ftz(s[mt][nt][j + 2] - mref);
                        ps += s[mt][nt][j] + s[mt][nt][j + 2];
                    }
                    l[nt][j] = fmaf(l[nt][j], alpha[nt][j], ps);
                }
            }
            if (__any_sync(FULL_MASK, grew)) {
#pragma unroll
                for (int dt = 0; dt < C::KS; ++dt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        acc[dt][nt][0] *= alpha[nt][0];
                        acc[dt][nt][1] *= alpha[nt][1];
                        acc[dt][nt][2] *= alpha[nt][0];
                        acc[dt][nt][3] *= alpha[nt][1];
                    }
            }

            // ---- O^T += V^T . P^T, P split into 16-bit hi + lo ----
#pragma unroll
            for (int mt = 0; mt < kMT; ++mt) {
                uint32_t bh[NT][2], bl[NT][2];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const float p0 = s[mt][nt][2 * hi], p1 = s[mt][nt][2 * hi + 1];
                        if constexpr (F8) {
                            const float h0 = f16_round(p0), h1 = f16_round(p1);
                            bh[nt][hi] = movmatrix_t(pack_f16(h0, h1));
                            bl[nt][hi] = movmatrix_t(pack_f16(p0 - h0, p1 - h1));
                        } else {
                            const float h0 = bf16_round(p0), h1 = bf16_round(p1);
                            bh[nt][hi] = movmatrix_t(pack_bf16(h0, h1));
                            bl[nt][hi] = movmatrix_t(pack_bf16(p0 - h0, p1 - h1));
                        }
                    }
                }
                if constexpr (F8) {
                    // this lane's token rows of the tile: grp (ldmatrix matrices
                    // 0, 2) and grp + 8 (matrices 1, 3); a row that does not take
                    // part is zeroed in registers (0-weight x NaN stays out)
                    bool ok_lo = true, ok_hi = true;
                    if (!whole) {
                        const int r0 = mt * 16 + grp, r1 = r0 + 8;
                        const int j0 = ((c * kCH + r0) >> p.log2_bs) - ((c * kCH) >> p.log2_bs);
                        const int j1 = ((c * kCH + r1) >> p.log2_bs) - ((c * kCH) >> p.log2_bs);
                        ok_lo = r0 < ntok && !((bad >> j0) & 1u);
                        ok_hi = r1 < ntok && !((bad >> j1) & 1u);
                    }
#pragma unroll
                    for (int j = 0; j < C::KS / 2; ++j) {
                        const int row = mt * 16 + k_row;
                        uint32_t r[4];
                        ldsm_x4(svb + row * D + (((2 * j + k_cx) ^ f8_swz<D>(row)) << 4), r);
                        if (!ok_lo) r[0] = r[2] = 0u;
                        if (!ok_hi) r[1] = r[3] = 0u;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            // m-tile dt = 2j + h: rows 0-7 the low code pairs, 8-15 the high
                            uint32_t xl, xh, yl, yh;
                            e4m3x4_to_f16(r[2 * h], xl, xh);      // tokens 0-7 of the tile
                            e4m3x4_to_f16(r[2 * h + 1], yl, yh);  // tokens 8-15
                            const uint32_t a[4] = {movmatrix_t(xl), movmatrix_t(xh), movmatrix_t(yl),
                                                   movmatrix_t(yh)};
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                mma_f16(acc[2 * j + h][nt], a, bh[nt][0], bh[nt][1]);
                                mma_f16(acc[2 * j + h][nt], a, bl[nt][0], bl[nt][1]);
                            }
                        }
                    }
                } else if constexpr (RC) {
                    // V^T by ldmatrix.trans over the rows of tile mt (tokens
                    // rc_token(mt, k)); a token that does not take part is
                    // zeroed in registers (k = 2 tig, 2 tig + 1 in a0/a1 and
                    // k + 8 in a2/a3)
                    const int tok = rc_token(mt, v_row, p.log2_bs);
                    const uint32_t rb = svb + (tok >> p.log2_bs) * rc_block_bytes<D>(p.block_size) +
                                        (tok & (p.block_size - 1)) * D * 2;
                    uint32_t keep0 = 0xffffffffu, keep1 = 0xffffffffu;
                    if (!whole) {
                        auto valid = [&](int k) {
                            const int t = rc_token(mt, k, p.log2_bs);
                            const int jrel = ((c * kCH + t) >> p.log2_bs) - ((c * kCH) >> p.log2_bs);
                            return t < ntok && !((bad >> jrel) & 1u);
                        };
                        keep0 = (valid(2 * tig) ? 0x0000ffffu : 0u) | (valid(2 * tig + 1) ? 0xffff0000u : 0u);
                        keep1 = (valid(2 * tig + 8) ? 0x0000ffffu : 0u) |
                                (valid(2 * tig + 9) ? 0xffff0000u : 0u);
                    }
#pragma unroll
                    for (int dt = 0; dt < C::KS; ++dt) {
                        uint32_t a[4];
                        ldsm_x4_t(rb + ((2 * dt + v_cx) << 4), a);
                        a[0] &= keep0;
                        a[1] &= keep0;
                        a[2] &= keep1;
                        a[3] &= keep1;
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma_bf16(acc[dt][nt], a, bh[nt][0], bh[nt][1]);
                            mma_bf16(acc[dt][nt], a, bl[nt][0], bl[nt][1]);
                        }
                    }
                } else {
#pragma unroll
                    for (int dt = 0; dt < C::KS; ++dt) {
                        const int half = dt >> 2;
                        const int chunk = (2 * (dt & 3) + v_cx) ^ r8;
                        uint32_t a[4];
                        ldsm_x4_t(svb + v_off[mt] + half * (128 << log2_rb) + (chunk << 4), a);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            mma_bf16(acc[dt][nt], a, bh[nt][0], bh[nt][1]);
                            mma_bf16(acc[dt][nt], a, bl[nt][0], bl[nt][1]);
                        }
                    }
                }
            }
            if (!F8 && !RC && !whole) fence_proxy_async_smem();  // our zero-fill before the next TMA write
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if constexpr (C::NCONS == 1) ring.advance(C::NSTAGE);
        }

        // ---- hand the segment's state to the epilogue warp ----
        // (a consumer that took no chunk of the segment hands over the
        // empty state)
        const int slot = me * S::NDUMP + dring.stage;
        if (!mbar_wait(&dempty[slot], dring.phase ^ 1u, p.wait_ns)) {
            if (lane == 0) {
                ctrl[0] = 1;
                raise_error(p.err, PKV_DEVERR_TIMEOUT);
            }
            return;
        }
        float* dump = reinterpret_cast<float*>(smem + S::OFF_DUMP + slot * S::DUMP_BYTES);
#pragma unroll
        for (int dt = 0; dt < C::KS; ++dt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) dump[((dt * NT + nt) * 4 + i) * 32 + lane] = acc[dt][nt][i];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                dump[(S::DUMP_ACC + nt * 4 + j) * 32 + lane] = m[nt][j];
                dump[(S::DUMP_ACC + nt * 4 + 2 + j) * 32 + lane] = l[nt][j];
            }
        __syncwarp();
        if (lane == 0) mbar_arrive(&dfull[slot]);
        dring.advance(S::NDUMP);
    }
}

// ---- shared-prefix results ------------------------------------------------------

// Tokens of request b's prefix group that the shared pass covered (0: none).
__device__ __forceinline__ int prefix_tokens_of(const DecodeParams& p, int b) {
    if (!p.prefix_of) return 0;
    const int g = __ldg(p.prefix_of + b);
    if (g < 0 || g >= p.num_prefixes) return 0;
    return prefix_tokens(p.prefix_lens, g, p.max_prefix_len, p.max_blocks * p.block_size,
                         p.log2_bs, p.err, false);
}

// A part's partial result (unnormalised acc, max m, sum l) in the record
// layout: acc rows of the 8*NT heads at `acc_rows`, their (m, l) pairs at
// `ml_rows` (global memory, or shared memory).
template <int D, int NT, bool F8>
__device__ __forceinline__ void store_frag(float* acc_rows, float* ml_rows, int tig, int grp,
                                           const float (&acc)[D / 16][NT][4],
                                           const float (&m)[NT][2], const float (&l)[NT][2]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int h = nt * 8 + 2 * tig + j;
            float* ra = acc_rows + h * D;
#pragma unroll
            for (int dt = 0; dt < D / 16; ++dt) {
                ra[dcol<F8>(dt, grp, 0)] = acc[dt][nt][j];
                ra[dcol<F8>(dt, grp, 1)] = acc[dt][nt][j + 2];
            }
            if (grp == 0) {
                ml_rows[h * 2] = m[nt][j];
                ml_rows[h * 2 + 1] = l[nt][j];
            }
        }
}

// ... as record `rec` of the workspace.
template <int D, int NT, bool F8>
__device__ __forceinline__ void write_record(const DecodeParams& p, size_t rec, int tig, int grp,
                                             const float (&acc)[D / 16][NT][4],
                                             const float (&m)[NT][2], const float (&l)[NT][2]) {
    constexpr int GP = 8 * NT;
    store_frag<D, NT, F8>(p.rec_acc + rec * GP * D, p.rec_ml + rec * GP * 2, tig, grp, acc, m, l);
}

// ---- epilogue: normalise, or write a partial record and merge the group ----

template <int D, int NT, bool F8, bool RC, bool SOLO>
__device__ __forceinline__ void epilogue(const DecodeParams& p, SegIter<kCH>& it,
                                         unsigned char* smem, uint64_t* dfull, uint64_t* dempty,
                                         volatile int* ctrl, int lane) {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    using S = Smem<D, NT, F8, SOLO, RC>;
    constexpr int GP = C::GP;
    const int grp = lane >> 2, tig = lane & 3;
    Ring dring;
    griddep_wait();  // `out` and the workspace may be in use by the previous kernel
    // Requests with no token at all: all-zero rows (softmax of an empty set).
    // (A request whose shared prefix covers all of it has no token of its own
    // pass either; the merge kernel writes it from the shared pass's results.)
    for (int b = blockIdx.x; b < p.num_seqs; b += gridDim.x) {
        if (clamp_len(p, b, false) != 0) continue;
        for (int i = lane; i < p.num_q_heads * D; i += 32)
            store_out(p.out, (size_t)b * p.num_q_heads * D + i, 0.f, p.out_dtype);
    }
    // A partial record (acc rows of GP heads, then their m/l pairs) as this
    // lane's fragment: from global memory (through L2), or from the
    // prefetch buffer in shared memory.
    auto load_frag = [&](const float* acc_rows, const float* ml_rows, bool global,
                         float (&mr)[NT][2], float (&lr)[NT][2], float (&ar)[C::KS][NT][4]) {
        auto ld = [&](const float* q) { return global ? ld_cg(q) : *q; };
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = nt * 8 + 2 * tig + j;
                const float* mlp = ml_rows + h * 2;
                const float* ra = acc_rows + h * D;
                mr[nt][j] = ld(mlp);
                lr[nt][j] = ld(mlp + 1);
#pragma unroll
                for (int dt = 0; dt < C::KS; ++dt) {
                    ar[dt][nt][j] = ld(ra + dcol<F8>(dt, grp, 0));
                    ar[dt][nt][j + 2] = ld(ra + dcol<F8>(dt, grp, 1));
                }
            }
    };
    auto load_rec = [&](size_t rec, float (&mr)[NT][2], float (&lr)[NT][2],
                        float (&ar)[C::KS][NT][4]) {
        load_frag(p.rec_acc + rec * GP * D, p.rec_ml + rec * GP * 2, true, mr, lr, ar);
    };
    // The epilogue warp is idle while the consumers stream a segment.  For a
    // group split over several units it watches, meanwhile, the ready flags of
    // the group's other parts (in merge order): a part that has seen all of
    // them is the last to finish without asking.  It also fetches the first
    // published record, so the merge's inputs are at hand: bf16 into
    // registers, fp8 (no registers to spare) into a shared-memory buffer with
    // asynchronous copies.  16-head groups neither watch nor prefetch.
    constexpr bool kWatch = NT == 1;
    constexpr bool kPrefetch = NT == 1 && !F8;
    constexpr bool kPrefetchSmem = S::PF_BYTES > 0;
    float* pf_acc = reinterpret_cast<float*>(smem + S::OFF_PF);
    float* pf_ml = pf_acc + GP * D;

    while (it.valid) {
        const Segment sg = it.current();
        it.advance(p, lane);
        const SegInfo si = seg_info<GP>(p, sg, it.W);
        const float vsc = F8 ? __ldg(p.v_scale + si.kvh) : 1.f;  // V dequantisation scale
        // Parts of the group: the records bg + u of its units u_first .. u_last.
        auto rec_of = [&](int k) -> size_t { return si.bg + (size_t)(si.u_first + k); };
        const int own = (int)(si.u - si.u_first);
        const bool split = !p.defer_merge && si.nseg > 1 && rec_of(si.nseg - 1) < (size_t)p.rec_cap;
        // next other part (ascending, skipping our own) whose flag has not been seen
        auto next_other = [&](int k) {
            ++k;
            if (k == own) ++k;
            return k;
        };
        int watch = split ? next_other(-1) : si.nseg;
        int pf_k = -1;  // the part whose record sits in pm / pl / pa
        float pm[NT][2], pl[NT][2], pa[C::KS][NT][4];

        // the segment's state: one consumer's, or the merge of NCONS consumers'
        float acc[C::KS][NT][4], m[NT][2], l[NT][2];
#pragma unroll
        for (int k = 0; k < C::NCONS; ++k) {
            const int slot = k * S::NDUMP + dring.stage;
            if constexpr (kWatch) {
                // Watch the flags until the hand-over is there: lane 0's flag
                // load is in flight while the warp tests the barrier.  Bounded
                // by the wait below, which also reports a hang.
                const uint64_t t0 = global_timer_ns();
                while (watch < si.nseg && !ctrl[0]) {
                    if (__any_sync(FULL_MASK, mbar_try_wait(&dfull[slot], dring.phase))) break;
                    unsigned f = 0u;
                    if (lane == 0) f = ld_acquire_u32(p.ready + rec_of(watch));
                    f = __shfl_sync(FULL_MASK, f, 0);
                    if (f) {
                        __syncwarp();  // lane 0's acquire orders the warp's reads of the record
                        if (pf_k < 0 && kPrefetch) {
                            load_rec(rec_of(watch), pm, pl, pa);
                            pf_k = watch;
                        } else if (pf_k < 0 && kPrefetchSmem) {
                            // the whole record, 16 bytes per copy, into the
                            // buffer (free once an earlier prefetch whose
                            // record went unused has landed)
                            cp_async_wait_all();
                            const float* ga = p.rec_acc + rec_of(watch) * GP * D;
                            const float* gm = p.rec_ml + rec_of(watch) * GP * 2;
                            for (int i = lane; i < GP * D / 4; i += 32) cp_async_cg16(pf_acc + 4 * i, ga + 4 * i);
                            if (lane < GP * 2 / 4) cp_async_cg16(pf_ml + 4 * lane, gm + 4 * lane);
                            pf_k = watch;
                        }
                        watch = next_other(watch);
                    }
                    if (global_timer_ns() - t0 > p.wait_ns) break;
                }
            }
            if (ctrl[0] || !mbar_wait(&dfull[slot], dring.phase, p.wait_ns)) {
                if (lane == 0 && !ctrl[0]) {
                    ctrl[0] = 1;
                    raise_error(p.err, PKV_DEVERR_TIMEOUT);
                }
                if constexpr (kPrefetchSmem) cp_async_wait_all();  // nothing lands after exit
                return;
            }
            const float* dump =
                reinterpret_cast<const float*>(smem + S::OFF_DUMP + slot * S::DUMP_BYTES);
            if (k == 0) {
#pragma unroll
                for (int dt = 0; dt < C::KS; ++dt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[dt][nt][i] = dump[((dt * NT + nt) * 4 + i) * 32 + lane];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        m[nt][j] = dump[(S::DUMP_ACC + nt * 4 + j) * 32 + lane];
                        l[nt][j] = dump[(S::DUMP_ACC + nt * 4 + 2 + j) * 32 + lane];
                    }
            } else {
                // combine with consumer k's state of the same segment (its
                // running max is common to the lanes of a head, like ours)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const float mk = dump[(S::DUMP_ACC + nt * 4 + j) * 32 + lane];
                        const float lk = dump[(S::DUMP_ACC + nt * 4 + 2 + j) * 32 + lane];
                        const float M = fmaxf(m[nt][j], mk);
                        const float mref = M == -INFINITY ? 0.f : M;
                        const float fa = exp2f(m[nt][j] - mref), fb = exp2f(mk - mref);
                        l[nt][j] = l[nt][j] * fa + lk * fb;
#pragma unroll
                        for (int dt = 0; dt < C::KS; ++dt) {
                            acc[dt][nt][j] = acc[dt][nt][j] * fa +
                                             dump[((dt * NT + nt) * 4 + j) * 32 + lane] * fb;
                            acc[dt][nt][j + 2] =
                                acc[dt][nt][j + 2] * fa +
                                dump[((dt * NT + nt) * 4 + j + 2) * 32 + lane] * fb;
                        }
                        m[nt][j] = M;
                    }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&dempty[slot]);
        }
        dring.advance(S::NDUMP);

        // the normaliser: sum the per-lane partials over the lanes sharing a head
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                l[nt][j] += __shfl_xor_sync(FULL_MASK, l[nt][j], 4);
                l[nt][j] += __shfl_xor_sync(FULL_MASK, l[nt][j], 8);
                l[nt][j] += __shfl_xor_sync(FULL_MASK, l[nt][j], 16);
            }
        if (p.defer_merge) {
            // Fixed partitions and prefix groups: every part of every group
            // publishes its record; the merge kernel combines them (with the
            // shared pass's results) in parallel.  The group's first part
            // tells it where the records are -- for every group with work, so
            // no stale word is ever read; a group that does not fit the
            // workspace is marked 0 and flagged, and the merge leaves it alone.
            const bool fits = si.bg + si.u_last < (size_t)p.rec_cap;
            if (si.u == si.u_first && lane == 0) {
                p.meta[2 * si.bg] = (int32_t)si.u_first;
                p.meta[2 * si.bg + 1] = fits ? si.nseg : 0;
                if (!fits) raise_error(p.err, PKV_DEVERR_BAD_SEQ_LEN);
            }
            if (fits) write_record<D, NT, F8>(p, si.bg + si.u, tig, grp, acc, m, l);
            continue;
        }
        if (si.nseg > 1 && !split) {
            if (lane == 0) raise_error(p.err, PKV_DEVERR_BAD_SEQ_LEN);
            continue;
        }
        if (split && watch < si.nseg) {
            // Not every other part is known to be out: arrive.  A part that
            // is not the last of its group to finish publishes its partial
            // result (record, then a release of its ready flag); the last one
            // keeps its own in registers and merges the others'.  (When every
            // other flag was seen, every other part has arrived and published:
            // this part is the last without asking.)
            unsigned arrived = 0;
            if (lane == 0) arrived = atomicAdd(p.counters + si.bg, 1u);
            arrived = __shfl_sync(FULL_MASK, arrived, 0);
            if (arrived != (unsigned)(si.nseg - 1)) {
                write_record<D, NT, F8>(p, rec_of(own), tig, grp, acc, m, l);
                __syncwarp();
                if (lane == 0) st_release_u32(p.ready + rec_of(own), 1u);
                continue;
            }

            // Last part: wait (bounded) until the remaining parts' records are out.
            int ok = 1;
            if (lane == 0) {
                const uint64_t t0 = global_timer_ns();
                for (int k = watch; k < si.nseg && ok; k = next_other(k)) {
                    for (uint32_t it = 0; ld_acquire_u32(p.ready + rec_of(k)) == 0u; ++it) {
                        if ((it & 63u) == 63u && global_timer_ns() - t0 > p.wait_ns) {
                            ok = 0;
                            break;
                        }
                    }
                }
                // (the test-only fault waits for the merger's own flag too,
                // which nothing sets)
                if (ok && p.fault_mode == kFaultMergeFlag) {
                    for (uint32_t it = 0; ld_acquire_u32(p.ready + rec_of(own)) == 0u; ++it) {
                        if ((it & 63u) == 63u && global_timer_ns() - t0 > p.wait_ns) {
                            ok = 0;
                            break;
                        }
                    }
                }
                if (!ok) raise_error(p.err, PKV_DEVERR_TIMEOUT);
            }
            ok = __shfl_sync(FULL_MASK, ok, 0);
            if (!ok) continue;
            __syncwarp();  // lane 0's acquires order the warp's reads of the records
        }
        // The row state: the group's parts merged in ascending part order
        // 0, 1, .., nseg - 1 whichever part finishes last, so the result does
        // not depend on timing.  Two states (m, l, acc) merge as M = max m,
        // l = 2^(m0-M) l0 + 2^(m1-M) l1, acc likewise, with separately
        // rounded products and one add, so the merge is symmetric in its
        // operands.  Records are fetched two at a time (8-head groups) with
        // every load of the pair in flight before any math.
        auto merge2 = [&](float (&m0)[NT][2], float (&l0)[NT][2], float (&a0)[C::KS][NT][4],
                          const float (&mr)[NT][2], const float (&lr)[NT][2],
                          const float (&ar)[C::KS][NT][4]) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const float M = fmaxf(m0[nt][j], mr[nt][j]);
                    const float mref = M == -INFINITY ? 0.f : M;
                    const float fa = exp2f(m0[nt][j] - mref), fb = exp2f(mr[nt][j] - mref);
                    l0[nt][j] = __fadd_rn(__fmul_rn(l0[nt][j], fa), __fmul_rn(lr[nt][j], fb));
#pragma unroll
                    for (int dt = 0; dt < C::KS; ++dt) {
                        a0[dt][nt][j] =
                            __fadd_rn(__fmul_rn(a0[dt][nt][j], fa), __fmul_rn(ar[dt][nt][j], fb));
                        a0[dt][nt][j + 2] = __fadd_rn(__fmul_rn(a0[dt][nt][j + 2], fa),
                                                      __fmul_rn(ar[dt][nt][j + 2], fb));
                    }
                    m0[nt][j] = M;
                }
        };
        // With a symmetric merge, this part's state, then the lowest other
        // part, then the rest in ascending order is the ascending order when
        // this part is part 0 or 1.  A later part first folds the parts below
        // it into a prefix.
        int k_from = 0;  // the first part the loop below considers
        if (split && own >= 2) {
            if constexpr (kPrefetch) {
                // bf16, 8-head groups: the prefix (parts 0 .. own-1) in the
                // prefetch registers, where part 0 may be already
                if (pf_k != 0) load_rec(rec_of(0), pm, pl, pa);
                for (int k = 1; k < own; ++k) {
                    float mr[NT][2], lr[NT][2], ar[C::KS][NT][4];
                    load_rec(rec_of(k), mr, lr, ar);
                    merge2(pm, pl, pa, mr, lr, ar);
                }
                merge2(m, l, acc, pm, pl, pa);
            } else {
                // No registers for a second state (fp8, 16-head groups): this
                // part's state goes out as its record too, the fold starts
                // from part 0 (fp8: from the shared-memory prefetch buffer
                // when it is there) and reads this part's record back in its
                // turn
                write_record<D, NT, F8>(p, rec_of(own), tig, grp, acc, m, l);
                __syncwarp();  // the m / l words are written by other lanes
                if (kPrefetchSmem && pf_k == 0) {
                    cp_async_wait_all();
                    __syncwarp();  // every lane's copies have landed
                    load_frag(pf_acc, pf_ml, false, m, l, acc);
                } else {
                    load_rec(rec_of(0), m, l, acc);
                }
                for (int k = 1; k <= own; ++k) {
                    float mr[NT][2], lr[NT][2], ar[C::KS][NT][4];
                    load_rec(rec_of(k), mr, lr, ar);
                    merge2(m, l, acc, mr, lr, ar);
                }
            }
            k_from = own + 1;
        } else {
            // the prefetched record is the lowest other part
            if (kPrefetch && split && pf_k >= 0) merge2(m, l, acc, pm, pl, pa);
            if (kPrefetchSmem && split && pf_k >= 0) {
                cp_async_wait_all();
                __syncwarp();  // every lane's copies have landed
                float mr[NT][2], lr[NT][2], ar[C::KS][NT][4];
                load_frag(pf_acc, pf_ml, false, mr, lr, ar);
                merge2(m, l, acc, mr, lr, ar);
            }
        }
        constexpr int kPair = NT == 1 ? 2 : 1;  // records in flight at once
        for (int k0 = k_from; split && k0 < si.nseg; k0 += kPair) {
            float mr[kPair][NT][2], lr[kPair][NT][2], ar[kPair][C::KS][NT][4];
            bool use[kPair];
#pragma unroll
            for (int k = 0; k < kPair; ++k) {
                const int kk = k0 + k;
                use[k] = kk < si.nseg && kk != own && kk != pf_k;
                if (use[k]) load_rec(rec_of(kk), mr[k], lr[k], ar[k]);
            }
#pragma unroll
            for (int k = 0; k < kPair; ++k)
                if (use[k]) merge2(m, l, acc, mr[k], lr[k], ar[k]);
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                const int h = nt * 8 + 2 * tig + j;
                if (h >= si.gv) continue;
                const float inv = l[nt][j] > 0.f ? vsc / l[nt][j] : 0.f;
                const size_t orow = ((size_t)si.b * p.num_q_heads + si.hq0 + h) * D;
#pragma unroll
                for (int dt = 0; dt < C::KS; ++dt) {
                    store_out(p.out, orow + dcol<F8>(dt, grp, 0), acc[dt][nt][j] * inv, p.out_dtype);
                    store_out(p.out, orow + dcol<F8>(dt, grp, 1), acc[dt][nt][j + 2] * inv,
                              p.out_dtype);
                }
            }
        if (split) {
            __syncwarp();
            if (lane == 0) {  // ready for the next call
                for (int k = 0; k < si.nseg; ++k) p.ready[rec_of(k)] = 0u;
                p.counters[si.bg] = 0u;
            }
        }
    }
    if constexpr (kPrefetchSmem) cp_async_wait_all();  // an unused prefetch lands before exit
}

// Total chunk count, computed by one warp (same value in every warp and CTA).
// *L_first / *T_first receive this lane's length of request `lane` and the
// first token of its pass (or 0).
__device__ __forceinline__ long long total_chunks_warp(const DecodeParams& p, int lane, bool flag,
                                                       int* L_first, int* T_first) {
    long long t = 0;
    *L_first = 0;
    *T_first = 0;
    for (int b = lane; b < p.num_seqs; b += 32) {
        const int L = clamp_len(p, b, flag);
        const int T = seq_begin(p, b, L, flag);
        if (b == lane) {
            *L_first = L;
            *T_first = T;
        }
        t += chunks_of<kCH>(L - T);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(FULL_MASK, t, off);
    return t * p.num_hg;
}

template <int D, int NT, bool F8, bool RC, bool SOLO, bool APP>
__global__ void __launch_bounds__(MmaCfg<D, NT, F8, SOLO, RC>::THREADS)
    decode_mma_kernel(const __grid_constant__ DecodeParams p,
                                                             const __grid_constant__ CUtensorMap tmk,
                                                             const __grid_constant__ CUtensorMap tmv) {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    using S = Smem<D, NT, F8, SOLO, RC>;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::OFF_BAR);
    uint64_t* empty = full + C::NSTAGE;
    uint64_t* dfull = empty + C::NSTAGE;
    uint64_t* dempty = dfull + S::NSLOT;
    int* st_ntok = reinterpret_cast<int*>(smem + S::OFF_META);
    unsigned* st_bad = reinterpret_cast<unsigned*>(st_ntok + C::NSTAGE);
    volatile int* ctrl = reinterpret_cast<volatile int*>(smem + S::OFF_CTRL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        ctrl[0] = 0;
        for (int s = 0; s < C::NSTAGE; ++s) {
            mbar_init(&full[s], 1);  // the producer's expect-tx arrival
            mbar_init(&empty[s], 1);  // released by the stage's one consumer
        }
        for (int s = 0; s < S::NSLOT; ++s) {
            mbar_init(&dfull[s], 1);
            mbar_init(&dempty[s], 1);
        }
        fence_mbar_init();
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
    }
    __syncthreads();
    griddep_launch_dependents();

    // Planning reads only seq_lens and the block tables, which the caller
    // guarantees are not produced by the kernel right before this one; so it
    // overlaps that kernel's tail.  Each role waits on the grid dependency
    // before touching K/V, q, out or the workspace.
    // The producer first guesses its first table window from the largest
    // length the caller announced (exact for a batch of equal lengths) and
    // starts loading it, so that load overlaps the seq_lens round trip.
    int spec_b = -1, spec_j = -1, spec_tab = -1;
    if (warp < C::NPROD && !p.prefix_of && p.fixed_units == 0 && p.max_len_hint > 0) {
        const int Lg = min(p.max_len_hint, p.max_blocks * p.block_size);
        const long long nchg = chunks_of<kCH>(Lg);
        const long long totg = nchg * p.num_hg * p.num_seqs;
        const long long Wg = (totg + gridDim.x - 1) / gridDim.x;
        const long long s0 = (long long)blockIdx.x * Wg;
        if (nchg > 0 && s0 < totg) {
            spec_b = (int)(s0 / (nchg * p.num_hg));
            spec_j = (int)((s0 % nchg) * kCH) >> p.log2_bs;
            const int nblkg = (Lg + p.block_size - 1) >> p.log2_bs;
            if (spec_j + lane < nblkg)
                spec_tab = __ldg(p.block_tables + (size_t)spec_b * p.max_blocks + spec_j + lane);
        }
    }
    int L_first = 0, T_first = 0;
    const long long total =
        total_chunks_warp(p, lane, blockIdx.x == 0 && warp == 0, &L_first, &T_first);
    if (total == 0) {
        if (warp == C::NPROD + C::NCONS) {
            SegIter<kCH> none;
            none.valid = false;
            epilogue<D, NT, F8, RC, SOLO>(p, none, smem, dfull, dempty, ctrl, lane);
        }
        return;
    }
    long long W = p.fixed_units > 0 ? p.fixed_units : (total + gridDim.x - 1) / gridDim.x;
    if (W < 1) W = 1;
    SegIter<kCH> it;
    it.init(p, total, W, lane, L_first, T_first);

    // warps: producers | consumers | epilogue
    if (warp < C::NPROD) {
        Producer<D, NT, F8, RC, SOLO, APP> pr{p, &tmk, &tmv, smem, full, empty, st_ntok, st_bad, ctrl, lane,
                           l2_policy_evict_first()};
        pr.me = warp;
        pr.run(it, spec_b, spec_j, spec_tab);
        if (!pr.waited) griddep_wait();
    } else if (warp < C::NPROD + C::NCONS) {
        consume<D, NT, F8, RC, SOLO>(p, it, smem, full, empty, dfull, dempty, st_ntok, st_bad, ctrl, lane,
                           warp - C::NPROD);
    } else {
        epilogue<D, NT, F8, RC, SOLO>(p, it, smem, dfull, dempty, ctrl, lane);
    }
}

// ---- deferred merge (fixed partitions, prefix groups) ---------------------------

constexpr int kMergeWarps = 4;  // warps that share one output row

// Merges output rows (request b, query head) over the parts of the row's own
// pass (records of the decode kernel) and the splits of its group's shared
// prefix pass.  RPC rows per CTA: with RPC == kMergeWarps each warp merges one
// row (many short rows: the grid fits one wave); with RPC == 1 the CTA's warps
// share one row, warp w taking records w, w + 4, ... (few long rows).  A warp
// reads its records eight at a time (each record row one coalesced run of
// float4 / float2, lane = head_dim/32 dims) and keeps a running max, sum and
// accumulator; the warps of a row meet in shared memory.
//   out = vscale * sum_r 2^(m_r - M) acc_r / sum_r 2^(m_r - M) l_r,  M = max_r m_r.
template <int D, int GP, int RPC>
__global__ void __launch_bounds__(32 * kMergeWarps)
    decode_mma_merge_kernel(const __grid_constant__ DecodeParams p) {
    constexpr int PER = D / 32;  // dims per lane
    constexpr int NB = 8;        // records in flight per warp
    constexpr int WPR = kMergeWarps / RPC;  // warps per row
    static_assert(RPC == 1 || RPC == kMergeWarps, "a row per CTA or a row per warp");
    __shared__ float red_acc[WPR > 1 ? kMergeWarps : 1][D];
    __shared__ float red_m[kMergeWarps], red_s[kMergeWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int wr = warp % WPR;  // this warp's rank among its row's warps
    const long long row = (long long)blockIdx.x * RPC + warp / WPR;
    const bool live = row < (long long)p.num_seqs * p.num_q_heads;
    const int b = live ? (int)(row / p.num_q_heads) : 0;
    const int hq = live ? (int)(row % p.num_q_heads) : 0;
    const int kvh = hq / p.group, jg = hq % p.group;
    const int hg = kvh * p.num_sub + jg / GP, h = jg % GP;
    const size_t bg = (size_t)b * p.num_hg + hg;
    const int L = live ? clamp_len(p, b, false) : 0;
    const int T = live ? seq_begin(p, b, L) : 0;
    const int ns = T > 0 ? prefix_num_splits(prefix_tokens_of(p, b), p.pfx_splits) : 0;
    griddep_wait();  // the records and meta of the kernels before
    // every condition below is the same in all threads of the row's warps
    int u0 = 0, nseg = 0;
    if (L > T) {
        u0 = p.meta[2 * bg];
        nseg = p.meta[2 * bg + 1];
        if (nseg == 0) return;  // did not fit the workspace (flagged by the decode kernel)
        if (u0 < 0 || (long long)bg + u0 + nseg > p.rec_cap) {  // never for a word this call wrote
            if (lane == 0 && wr == 0) raise_error(p.err, PKV_DEVERR_BAD_SEQ_LEN);
            return;
        }
    }
    const int n = nseg + ns;
    if (n == 0) return;  // an empty request (or no row): the decode kernel wrote zeros
    const size_t rec0 = bg + u0;
    // record r < nseg: own part r; r >= nseg: split r - nseg of the shared pass
    auto ml_of = [&](int r) -> const float* {
        return r < nseg ? p.rec_ml + ((rec0 + r) * GP + h) * 2
                        : p.pfx_ml + (((size_t)(r - nseg) * p.num_seqs + b) * p.num_q_heads + hq) * 2;
    };
    auto acc_of = [&](int r) -> const float* {
        return r < nseg ? p.rec_acc + ((rec0 + r) * GP + h) * D
                        : p.pfx_acc + (((size_t)(r - nseg) * p.num_seqs + b) * p.num_q_heads + hq) * D;
    };
    auto load_row = [&](const float* acc, float (&v)[PER]) {
        if constexpr (PER == 4) {
            const float4 t = *reinterpret_cast<const float4*>(acc + lane * 4);
            v[0] = t.x;
            v[1] = t.y;
            v[2] = t.z;
            v[3] = t.w;
        } else {
            const float2 t = *reinterpret_cast<const float2*>(acc + lane * 2);
            v[0] = t.x;
            v[1] = t.y;
        }
    };
    // this warp's records, NB at a time (the last batch predicated)
    float A[PER], S = 0.f, mw = -INFINITY;
#pragma unroll
    for (int i = 0; i < PER; ++i) A[i] = 0.f;
    for (int r0 = wr; r0 < n; r0 += WPR * NB) {
        float v[NB][PER], mm[NB], ll[NB];
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const int r = r0 + WPR * q;
            if (r < n) {
                const float* ml = ml_of(r);
                mm[q] = ml[0];
                ll[q] = ml[1];
                load_row(acc_of(r), v[q]);
            } else {
                mm[q] = -INFINITY;
                ll[q] = 0.f;
#pragma unroll
                for (int i = 0; i < PER; ++i) v[q][i] = 0.f;
            }
        }
        float mb = mw;
#pragma unroll
        for (int q = 0; q < NB; ++q) mb = fmaxf(mb, mm[q]);
        const float ref = mb == -INFINITY ? 0.f : mb;
        const float c = exp2f(mw - ref);  // 0 while nothing is held
        S *= c;
#pragma unroll
        for (int i = 0; i < PER; ++i) A[i] *= c;
#pragma unroll
        for (int q = 0; q < NB; ++q) {
            const float wq = exp2f(mm[q] - ref);
            S = fmaf(ll[q], wq, S);
#pragma unroll
            for (int i = 0; i < PER; ++i) A[i] = fmaf(v[q][i], wq, A[i]);
        }
        mw = mb;
    }
    const float vsc = p.v_scale ? __ldg(p.v_scale + kvh) : 1.f;
    const size_t orow = ((size_t)b * p.num_q_heads + hq) * D + lane * PER;
    if constexpr (WPR == 1) {
        const float inv = S > 0.f ? vsc / S : 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) store_out(p.out, orow + i, A[i] * inv, p.out_dtype);
    } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) red_acc[warp][lane * PER + i] = A[i];
        if (lane == 0) {
            red_m[warp] = mw;
            red_s[warp] = S;
        }
        __syncthreads();
        if (warp != 0) return;
        float M = red_m[0];
#pragma unroll
        for (int w = 1; w < kMergeWarps; ++w) M = fmaxf(M, red_m[w]);
        const float ref = M == -INFINITY ? 0.f : M;
        float cw[kMergeWarps], St = 0.f;
#pragma unroll
        for (int w = 0; w < kMergeWarps; ++w) {
            cw[w] = exp2f(red_m[w] - ref);
            St = fmaf(red_s[w], cw[w], St);
        }
        const float inv = St > 0.f ? vsc / St : 0.f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            float t = 0.f;
#pragma unroll
            for (int w = 0; w < kMergeWarps; ++w) t = fmaf(red_acc[w][lane * PER + i], cw[w], t);
            store_out(p.out, orow + i, t * inv, p.out_dtype);
        }
    }
}

// ---- host side ---------------------------------------------------------------

template <int D, int NT, bool F8, bool RC, bool SOLO, bool APP = false>
pkv_status launch_impl(const DecodeParams& p, cudaStream_t stream, int* grid_out) {
    using C = MmaCfg<D, NT, F8, SOLO, RC>;
    using S = Smem<D, NT, F8, SOLO, RC>;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    static std::mutex mu;
    static int occupancy[64] = {0};
    auto kern = decode_mma_kernel<D, NT, F8, RC, SOLO, APP>;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (di->device >= 64) return PKV_ERR_UNSUPPORTED;
        if (occupancy[di->device] == 0) {
            if (S::BYTES > di->max_smem_optin) return PKV_ERR_UNSUPPORTED;
            if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S::BYTES) !=
                cudaSuccess)
                return PKV_ERR_CUDA;
            int occ = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, C::THREADS, S::BYTES) !=
                    cudaSuccess ||
                occ < 1)
                return PKV_ERR_CUDA;
            occupancy[di->device] = occ;
        }
    }
    const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
    const int box_rows = std::min(p.block_size, kCH);
    CUtensorMap tmk, tmv;
    if (!encode_cache_map(&tmk, p.k_cache, rows, D, box_rows, F8, !F8 && !RC) ||
        !encode_cache_map(&tmv, p.v_cache, rows, D, box_rows, F8, !F8 && !RC))
        return PKV_ERR_CUDA;
    const int grid = di->num_sms * std::min(occupancy[di->device], 4);

    PdlLaunch L(dim3(grid), dim3(C::THREADS), S::BYTES, stream);
    if (cudaLaunchKernelEx(&L.cfg, kern, p, tmk, tmv) != cudaSuccess) return PKV_ERR_CUDA;
    if (p.defer_merge) {
        constexpr int GP = MmaCfg<D, NT, F8>::GP;
        // many rows: one warp per row (a single wave of CTAs); few rows, which
        // may each hold many parts: the CTA's warps share a row
        const long long rows = (long long)p.num_seqs * p.num_q_heads;
        const bool per_warp = rows >= 4LL * di->num_sms;
        const long long mgrid = per_warp ? (rows + kMergeWarps - 1) / kMergeWarps : rows;
        if (mgrid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
        PdlLaunch M(dim3((unsigned)mgrid), dim3(32 * kMergeWarps), 0, stream);
        const cudaError_t e =
            per_warp ? cudaLaunchKernelEx(&M.cfg, decode_mma_merge_kernel<D, GP, kMergeWarps>, p)
                     : cudaLaunchKernelEx(&M.cfg, decode_mma_merge_kernel<D, GP, 1>, p);
        if (e != cudaSuccess) return PKV_ERR_CUDA;
    }
    if (grid_out) *grid_out = grid;
    return PKV_OK;
}

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

namespace {

// The last few views encoded, so that a caller decoding the same caches call
// after call (every layer of a serving loop) pays for encoding once.
struct MapCacheEntry {
    const void* base = nullptr;
    long long rows = 0;
    int head_dim = 0, box_rows = 0;
    bool fp8 = false, both_halves = false;
    CUtensorMap map;
};
constexpr int kMapCache = 16;
std::mutex g_map_mu;
MapCacheEntry g_map_cache[kMapCache];
int g_map_next = 0;

}  // namespace

// 2-D view of a cache: rows = num_blocks*Hkv*block_size, columns = head_dim
// bf16; boxes of 64 columns x min(block_size, 64) rows, 128-byte swizzle.
// both_halves (bf16, head_dim 128): a 3-D view (64 columns, rows, 2 halves
// 128 bytes apart) whose boxes hold both halves of box_rows rows, landing as
// [half][row][128 B].  fp8: rows of head_dim one-byte codes, whole-row boxes
// with the swizzle of their width (128 bytes at head_dim 128, 64 at 64),
// which the consumers' reads apply.
bool encode_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim,
                      int box_rows, bool fp8, bool both_halves) {
    both_halves = both_halves && !fp8 && head_dim == 128;
    {
        std::lock_guard<std::mutex> lock(g_map_mu);
        for (const MapCacheEntry& e : g_map_cache)
            if (e.base == base && e.rows == rows && e.head_dim == head_dim &&
                e.box_rows == box_rows && e.fp8 == fp8 && e.both_halves == both_halves) {
                *map = e.map;
                return true;
            }
    }
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t row_bytes = (cuuint64_t)head_dim * (fp8 ? 1 : 2);
    cuuint64_t gdim[3] = {(cuuint64_t)(both_halves ? 64 : head_dim), (cuuint64_t)rows, 2};
    cuuint64_t gstride[2] = {row_bytes, 128};
    cuuint32_t box[3] = {fp8 ? (cuuint32_t)head_dim : 64u, (cuuint32_t)box_rows, 2u};
    cuuint32_t estride[3] = {1u, 1u, 1u};
    const CUresult r = enc(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                           both_halves ? 3 : 2, const_cast<void*>(base), gdim, gstride, box,
                           estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           (fp8 && head_dim == 64) ? CU_TENSOR_MAP_SWIZZLE_64B
                                                   : CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    std::lock_guard<std::mutex> lock(g_map_mu);
    MapCacheEntry& e = g_map_cache[g_map_next];
    g_map_next = (g_map_next + 1) % kMapCache;
    e.base = base;
    e.rows = rows;
    e.head_dim = head_dim;
    e.box_rows = box_rows;
    e.fp8 = fp8;
    e.both_halves = both_halves;
    e.map = *map;
    return true;
}

bool decode_mma_supported(int head_dim, int block_size, pkv_dtype q_dtype, pkv_dtype kv_dtype) {
    // blocks of >= 8 rows: TMA boxes; bf16 blocks of 2 or 4 rows: per-lane row copies
    // (a 64-token chunk then spans 32 or 16 blocks, within one table window)
    const bool rows_ok = block_size >= 8 ||
                         (kv_dtype == PKV_BF16 && (block_size == 2 || block_size == 4));
    return q_dtype == PKV_BF16 && (kv_dtype == PKV_BF16 || kv_dtype == PKV_FP8_E4M3) &&
           (head_dim == 64 || head_dim == 128) && rows_ok;
}

// bf16 caches: TMA boxes or row copies, one CTA per SM or two (SOLO), with or
// without the fused append.
template <bool APP>
pkv_status launch_bf16(const DecodeParams& p, int head_dim, int nt, bool many, cudaStream_t stream,
                       int* grid_out) {
    if constexpr (APP) {
        // the append rides only in the one-CTA-per-SM layout (decode_mma_fuses_append)
        if (nt == 2 || many) return PKV_ERR_UNSUPPORTED;
        if (head_dim == 128)
            return p.row_copy ? launch_impl<128, 1, false, true, false, true>(p, stream, grid_out)
                              : launch_impl<128, 1, false, false, false, true>(p, stream, grid_out);
        if (head_dim == 64)
            return p.row_copy ? launch_impl<64, 1, false, true, false, true>(p, stream, grid_out)
                              : launch_impl<64, 1, false, false, false, true>(p, stream, grid_out);
        return PKV_ERR_UNSUPPORTED;
    }
    if (p.row_copy) {
        if (head_dim == 128)
            return nt == 2 ? launch_impl<128, 2, false, true, true, APP>(p, stream, grid_out)
                   : many  ? launch_impl<128, 1, false, true, true, APP>(p, stream, grid_out)
                           : launch_impl<128, 1, false, true, false, APP>(p, stream, grid_out);
        if (head_dim == 64)
            return nt == 2 ? launch_impl<64, 2, false, true, true, APP>(p, stream, grid_out)
                   : many  ? launch_impl<64, 1, false, true, true, APP>(p, stream, grid_out)
                           : launch_impl<64, 1, false, true, false, APP>(p, stream, grid_out);
    } else {
        if (head_dim == 128)
            return nt == 2 ? launch_impl<128, 2, false, false, true, APP>(p, stream, grid_out)
                   : many  ? launch_impl<128, 1, false, false, true, APP>(p, stream, grid_out)
                           : launch_impl<128, 1, false, false, false, APP>(p, stream, grid_out);
        if (head_dim == 64)
            return nt == 2 ? launch_impl<64, 2, false, false, true, APP>(p, stream, grid_out)
                   : many  ? launch_impl<64, 1, false, false, true, APP>(p, stream, grid_out)
                           : launch_impl<64, 1, false, false, false, APP>(p, stream, grid_out);
    }
    return PKV_ERR_UNSUPPORTED;
}

// Many (request, head group) pairs: at least four per SM.  Then two CTAs per
// SM (one consumer and one epilogue warp each) share the many short segments
// better than one CTA with two consumers.
static bool many_groups(const DecodeParams& p, int num_sms) {
    return (long long)p.num_seqs * p.num_hg >= 4LL * num_sms;
}

bool decode_mma_fuses_append(const DecodeParams& p, int group_pad) {
    const DeviceInfo* di = current_device_info();
    return di && group_pad <= 8 && !many_groups(p, di->num_sms);
}

pkv_status launch_decode_mma(const DecodeParams& p, int head_dim, int group_pad, bool fp8,
                             cudaStream_t stream, int* grid_out) {
    const int nt = group_pad > 8 ? 2 : 1;
    // bf16, 8-head groups: one CTA per SM with two consumers, unless the call
    // has at least four (request, head group) pairs per SM --
    // then few of them split, and two CTAs per SM (one consumer and one
    // epilogue warp each) share the many short segments better.
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    const bool many = many_groups(p, di->num_sms);
    if (fp8) {
        if (p.row_copy) return PKV_ERR_UNSUPPORTED;
        if (head_dim == 128) return nt == 1 ? launch_impl<128, 1, true, false, false>(p, stream, grid_out)
                                            : launch_impl<128, 2, true, false, false>(p, stream, grid_out);
        if (head_dim == 64) return nt == 1 ? launch_impl<64, 1, true, false, false>(p, stream, grid_out)
                                           : launch_impl<64, 2, true, false, false>(p, stream, grid_out);
    } else if (p.k_new) {
        return launch_bf16<true>(p, head_dim, nt, many, stream, grid_out);
    } else {
        return launch_bf16<false>(p, head_dim, nt, many, stream, grid_out);
    }
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace pkv
