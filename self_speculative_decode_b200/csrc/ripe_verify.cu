// Verification attention over a RIPE multi-plane KV cache (sm_100a).
//
// What is computed (RIPE abstract, "Prefix Keys and Values Matter Late: RIPE Caching for
// Self-Speculative Decoding in Looped Language Models", first, fourth and fifth sentences):
// for every query head of every draft-block position p = T + j at loop r, the causal
// softmax attention over keys t <= p, where a key reads plane r when it belongs to the
// draft block or to the window, and the shared deepest plane R-1 otherwise.
//
// How (one persistent launch per call):
//   * The keys of each (sequence, kv head) form a tile list: deepest-plane tiles, ring tiles
//     at plane r, and at most two "dual" ring tiles at plane R-1 holding the window keys
//     that later queries of the block see at the deepest plane (query-relative window).
//     All lists are concatenated and cut into equal contiguous chunks, one per CTA, so
//     ragged lengths and the three layouts (full, RIPE, deepest-only) balance the same way;
//     when every head has the same tile count and there are fewer heads than CTAs, each
//     head is cut into equal pieces instead, one per CTA, so that no CTA straddles two heads.
//   * One producer thread streams 64-key K/V tiles with 3-D TMA loads (64-byte swizzle, no
//     multicast) into a shared-memory ring of NS stages guarded by mbarriers, and writes a
//     small descriptor of each tile (sequence, kv head, kind, first key, count) beside it.
//     For two query tiles per warp its warp heads a warpgroup of its own that gives registers
//     up (setmaxnreg) to the two consumer warpgroups, so that their fragments of Q, O and S fit
//     without spilling.
//   * Consumer warps work on the transposed problem S^T = K Q^T (keys on the MMA's M side,
//     the B x group query rows on its N side, so an 8-row block is not padded to 16), with
//     mma.sync m16n8k16 bf16 -> fp32.  P^T is moved into the B-operand layout of
//     O^T += V^T P^T with movmatrix.  Every query row of one kv head is served by the same
//     K/V tile (GQA group sharing).  Two groups of warps consume alternate tiles.
//   * Online softmax in base 2; the reference maximum only moves when a tile's maximum
//     exceeds it by more than 8 (so probabilities stay <= 2^8), which skips most O rescales
//     and is exact.  Full deepest-plane tiles take a path without masks.
//   * A CTA that covers a whole (sequence, kv head) writes the output directly.  A head cut
//     into two pieces is held by the two CTAs of a cluster: the second sends its unnormalised
//     partial (o, m, l) into the first's shared memory (st.async counted on an mbarrier) and
//     the first merges the two by log-sum-exp.  Otherwise the CTAs write partials to global
//     scratch; the last to arrive (atomic counter, no spinning) merges them.
//   * Every wait is bounded: on timeout the kernel records RIPE_DEVERR_WAIT_TIMEOUT, drains
//     its own copies in flight and returns without writing further results.
#include <atomic>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "ripe_verify.cuh"

namespace ripe {

// Query-side shapes: NQT 8-query tiles per warp, WR row groups, WK key groups per tile,
// TG tile groups consuming alternate tiles.
template <int D, int NQT, int WR, int WK, int TG>
struct VCfg {
    static constexpr int NQ = 8 * NQT;             // queries per warp
    static constexpr int ROWS = NQ * WR;           // query rows per (sequence, kv head)
    static constexpr int GW = WR * WK;             // warps per tile group
    static constexpr int NCW = GW * TG;            // consumer warps
    // Threads: the consumers, the producer warp and (fused form) the copy warp.  With two query
    // tiles per warp (SPLIT), whose Q, O and S fragments do not fit the 168 registers that three
    // warps per sub-partition leave, the producer and copy warps are padded to a warpgroup that
    // gives registers up (setmaxnreg) to the consumer warpgroups: launched at LAUNCH_REGS per
    // thread, they run at REG_CONSUMER, the producer group at REG_PRODUCER, and the split adds up
    // to no more than the launch's registers.  Without it a CTA keeps enough registers free for a
    // small kernel (the append) to share the SM.
    static constexpr bool SPLIT = NQT >= 2;
    static constexpr int THREADS = SPLIT ? (NCW + 4) * 32 : (NCW + 1) * 32;
    static constexpr int threads(bool fused) { return THREADS + (fused && !SPLIT ? 32 : 0); }
    static constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8 > 255 ? 248 : (65536 / THREADS) / 8 * 8;
    static constexpr int REG_PRODUCER = 72;
    static constexpr int REG_CONSUMER =
        ((LAUNCH_REGS * (NCW + 4) - 4 * REG_PRODUCER) / NCW) / 8 * 8 > 248
            ? 248
            : ((LAUNCH_REGS * (NCW + 4) - 4 * REG_PRODUCER) / NCW) / 8 * 8;
    static_assert(NCW % 4 == 0, "consumer warps form whole warpgroups");
    static_assert(NCW * REG_CONSUMER + 4 * REG_PRODUCER <= (NCW + 4) * LAUNCH_REGS, "register split");
    static constexpr int SB = 4 / WK;              // 16-key sub-blocks per warp per tile
    static constexpr int NBOX = D / kBoxCols;
    static constexpr int STAGE_BYTES = 2 * NBOX * kBoxBytes;
    static constexpr int DP = D + 4;               // merge-buffer row stride (no bank conflicts)
    static constexpr int MERGE_FLOATS = NCW * NQ * DP;
    // receive buffer of the cluster-pair merge: the partner's o [ROWS][D] and (m, l) [ROWS][2]
    static constexpr bool XPAIR = ROWS <= 16;
    static constexpr int XF = XPAIR ? ROWS * D + 4 * ROWS : 0;
    // per (warp, query) and per row: (m, l_out, l_lse, -), see the softmax below
    static constexpr int MLF = NCW * NQ * 4 + ROWS * (TG * WK + 4) + XF;
    static constexpr int MISC = 1024 /*align*/ + 1024 /*bars, descriptors, flags*/;
    static constexpr int AVAIL = kSmemLimit - MISC - 4 * (MERGE_FLOATS + MLF) - 4 * (2 * kMaxBatch + 2);
    static constexpr int CAP = (D == 128 && TG == 1) ? RIPE_MAX_STAGES_WIDE : RIPE_MAX_STAGES;
    static constexpr int NS_RAW = AVAIL / STAGE_BYTES > CAP ? CAP : AVAIL / STAGE_BYTES;
    // A multiple of TG: a stage's previous tile then belongs to the same tile group, whose wait on
    // it has completed.  With a stage shared by both groups, a group could wait on a tile whose
    // stage still carries the other group's older tile in flight; the parity test would pass one
    // phase early and the group would read that tile's data and descriptor.
    static constexpr int NS = NS_RAW - NS_RAW % TG;
    static_assert(NS >= 2, "not enough shared memory for the pipeline");
    static constexpr int SMEM_FIXED = MISC + NS * STAGE_BYTES + 4 * (MERGE_FLOATS + MLF);
    // the end-of-CTA merge keeps m and l of every partial of a query row in the stage buffers:
    // at most MAX_PARTS partials, so at most MAX_PARTS CTAs (enough for a 148-SM B200)
    static constexpr int MAX_PARTS = (NS * STAGE_BYTES) / (2 * ROWS * 4) < 256 ? (NS * STAGE_BYTES) / (2 * ROWS * 4) : 256;
#ifndef RIPE_ALLOW_SMALL_GRID
    static_assert(MAX_PARTS >= 148, "stage buffers too small for the end-of-CTA merge");
#endif
};

template <class C>
__host__ __device__ constexpr int smem_bytes_for(int N) {
    return C::SMEM_FIXED + (2 * N + 2) * 4;
}

// Fused append: the rows of the draft block (positions >= T + j0) inside this CTA's ring tiles
// are copied from the caller's block K/V [N][qB][kvH][d] into ring plane r.  No other tile of
// the launch reads those slots.  Kept out of line: it runs once per CTA, away from the tile loop.
template <int D>
__device__ __noinline__ void fused_block_copy(const VerifyArgs &a, const int *cum, const int *Ts, int g_begin,
                                              int g_end, int tid, int nthreads) {
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;
    const int p_first = pair_of(cum, N, kvH, g_begin), p_last = pair_of(cum, N, kvH, g_end - 1);
    const int d8 = D / 8;
    for (int p = p_first; p <= p_last; ++p) {
        const int n = p / kvH, kh = p - (p / kvH) * kvH;
        const SeqGeom sg = seq_geom(Ts[n], pa);
        if (sg.T + a.B > a.max_T) {
            if (tid == 0) atomicOr(a.err, RIPE_DEVERR_CAPACITY);
            continue;
        }
        const int start = cum[n] + kh * sg.total;
        const int first = sg.T + a.j0;  // first position written by this call
        const int lt_hi = ring_tile_of(sg, pa, sg.T + a.B - 1);
        for (int lt = ring_tile_of(sg, pa, first); lt <= lt_hi; ++lt) {
            const int gt = start + lt;
            if (gt < g_begin || gt >= g_end) continue;
            const Tile t = tile_at(sg, lt, pa);
            const int r0 = t.t0 > first ? t.t0 : first;
            const int rows = t.t0 + t.cnt - r0;
            for (int e = tid; e < rows * d8; e += nthreads) {
                const int row = e / d8, c8 = e - (e / d8) * d8;
                const int tpos = r0 + row;
                const size_t src = ((static_cast<size_t>(n) * a.qB + (tpos - first)) * kvH + kh) * d8 + c8;
                const size_t dst = ((((static_cast<size_t>(a.layer) * N + n) * a.R + t.plane) * kvH + kh) *
                                        pa.ring_slots + (t.y + (tpos - t.t0))) * d8 + c8;
                a.ring_k[dst] = a.blk_k[src];
                a.ring_v[dst] = a.blk_v[src];
            }
        }
    }
}

// Fused append: index (within the chunk) of the first tile holding a row the launch writes
// (positions T + j0 .. T + B - 1 of a pair), or ntiles if the chunk has none.  The chunk
// starts at tile lt of pair (n, kh) with geometry sg.
__device__ __noinline__ int first_written_tile(SeqGeom sg, int lt, int n, int kh, int ntiles, const int *Ts,
                                               const VerifyArgs &a) {
    const PlanArgs &pa = a.plan;
    int i = 0;
    while (i < ntiles) {
        const int lo = ring_tile_of(sg, pa, sg.T + a.j0), hi = ring_tile_of(sg, pa, sg.T + a.B - 1);
        if (lt <= hi) {
            const int at = i + (lo > lt ? lo - lt : 0);
            return at < ntiles ? at : ntiles;
        }
        i += sg.total - lt;
        lt = 0;
        if (++kh == a.kvH) {
            kh = 0;
            if (++n >= a.N) break;
            sg = seq_geom(Ts[n], pa);
        }
    }
    return ntiles;
}

// FUSED adds one warp after the producer that writes the draft block's rows into the ring.
template <int D, int NQT, int WR, int WK, int TG, bool FUSED>
__global__ void __launch_bounds__(VCfg<D, NQT, WR, WK, TG>::threads(FUSED), 1)
ripe_verify_kernel(const __grid_constant__ CUtensorMap tmKd, const __grid_constant__ CUtensorMap tmVd,
                   const __grid_constant__ CUtensorMap tmKw, const __grid_constant__ CUtensorMap tmVw,
                   const __grid_constant__ VerifyArgs a) {
    using C = VCfg<D, NQT, WR, WK, TG>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stages = base;
    float *mo = reinterpret_cast<float *>(base + NS * C::STAGE_BYTES);   // [NCW][NQ][DP]
    float *mml = mo + C::MERGE_FLOATS;                                   // [NCW][NQ][4] m, l_out, l_lse
    float *wq = mml + C::NCW * C::NQ * 4;                                // [ROWS][TG*WK] weights
    float *fin = wq + C::ROWS * TG * WK;                                 // [ROWS][4] final M, L_out, L_lse
    float *xo = fin + C::ROWS * 4;                                       // [ROWS][D] partner's o (XPAIR)
    float *xml = xo + C::ROWS * D;                                       // [ROWS][4] partner's M, L_out, L_lse
    uint64_t *bars = reinterpret_cast<uint64_t *>(mml + C::MLF);         // full[NS], empty[NS], block
    TileDesc *sdesc = reinterpret_cast<TileDesc *>(bars + 2 * NS + 2);   // [NS]
    int *sflag = reinterpret_cast<int *>(sdesc + NS);                    // [16]
    int *cum = sflag + 16;                                               // [N + 1]
    int *Ts = cum + a.N + 1;                                             // [N]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;

    if (warp == C::NCW && lane == 0) {  // descriptors are parameters: fetch them before the wait
        tma_prefetch_desc(&tmKw);
        tma_prefetch_desc(&tmVw);
        if (a.has_deep) {
            tma_prefetch_desc(&tmKd);
            tma_prefetch_desc(&tmVd);
        }
    }
    if (tid == 0) {
        sflag[1] = 0;  // abort flag
        sflag[3] = 0;  // pairs this CTA merges at the end (at most its first and last): sflag[4..5]
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_addr(&bars[s]), 1);
            mbar_init(smem_addr(&bars[NS + s]), C::GW);
        }
        if (FUSED) mbar_init(smem_addr(&bars[2 * NS]), 1);  // draft block written into the ring
        if (C::XPAIR && a.xpair) {
            // partner's partial received: the first CTA of a pair expects its bytes (used only
            // when the pair splits one head; otherwise nothing waits on it)
            mbar_init(smem_addr(&bars[2 * NS + 1]), 1);
            if (!(blockIdx.x & 1)) mbar_expect_tx(smem_addr(&bars[2 * NS + 1]), a.Mq * (D * 4 + 16));
        }
        mbar_fence_init();
    }
    // the partner may arrive on this CTA's barrier: both CTAs of the pair initialise theirs first
    if (C::XPAIR && a.xpair) cluster_sync_all();
    // rows past a short box are never written by TMA: keep them finite
    if (pa.deep_box < kTileRows || pa.ring_box < kTileRows) {
        uint4 *z = reinterpret_cast<uint4 *>(stages);
        for (int i = tid; i < NS * C::STAGE_BYTES / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    }
    // ---- per-sequence tile counts and their prefix sums (T is written by earlier kernels)
    if (!a.early) pdl_wait();
    const ChunkPlan cp = plan_chunks(a, cum, Ts, sflag, tid, warp, lane);
    const int chunk = cp.chunk, pieces = cp.pieces, head = cp.head;
    const int g_begin = cp.g_begin, g_end = cp.g_end;
    const SeqGeom &sg1 = cp.sg1;
    if (g_begin >= g_end) {
        if (a.early) pdl_wait();  // the launch completes only after its predecessor
        return;
    }
    const int ntiles = g_end - g_begin;
    // (sequence, kv head) pairs of this CTA's first and last tiles
    const int P_first = pieces ? head : pair_of(cum, N, kvH, g_begin);
    const int P_last = pieces ? head : pair_of(cum, N, kvH, g_end - 1);

    const uint32_t full0 = smem_addr(&bars[0]);
    const uint32_t empty0 = smem_addr(&bars[NS]);
    const uint32_t stage0 = smem_addr(stages);

    // FUSED (ripe_append_verify, draft steps): a copy warp writes the block rows into the ring; a
    // separate instantiation so that plain verification carries none of that code
    constexpr bool fused = FUSED;
    if (warp >= C::NCW) {
        // the producer warpgroup hands registers to the consumers
        if constexpr (C::SPLIT) setmaxnreg_dec<C::REG_PRODUCER>();
        if constexpr (fused) {
            if (warp == C::NCW + 1) {
                // the copy warp: write the draft block's rows that this CTA's tiles read into the
                // ring, fence them for the TMA (async proxy), release the producer
                if (a.early) pdl_wait();  // the caller's block rows and the ring slots they replace
                fused_block_copy<D>(a, cum, Ts, g_begin, g_end, lane, 32);
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bars[2 * NS]));
                return;
            }
        }
        if (warp != C::NCW) return;
        // ================================================================ producer (one thread)
        if (lane != 0 && a.early) {
            // the other lanes bring the first pair's query rows into L2 while the previous launch
            // finishes (the consumers load them once it has)
            const int n0 = P_first / kvH, kh0 = P_first - n0 * kvH;
            for (int i = lane - 1; i < a.Mq; i += 31) {
                const int j = i / a.g, hg = i - j * a.g;
                const char *row = reinterpret_cast<const char *>(
                    a.q + ((static_cast<size_t>(n0) * a.qB + j) * a.Hq + kh0 * a.g + hg) * D);
                for (int off = 0; off < D * 2; off += 128) asm volatile("prefetch.global.L2 [%0];" ::"l"(row + off));
            }
        }
        if (lane == 0) {
            int n, kh, lt;
            SeqGeom sg;
            if (pieces) {  // one head per CTA: no search, no division by the head's tile count
                n = N == 1 ? 0 : P_first / kvH;
                kh = P_first - n * kvH;
                sg = N == 1 ? sg1 : seq_geom(Ts[n], pa);
                lt = (blockIdx.x - head * pieces) * chunk;
            } else {
                n = seq_of(cum, N, g_begin);
                sg = seq_geom(Ts[n], pa);
                const int rel = g_begin - cum[n];
                kh = rel / sg.total;
                lt = rel - kh * sg.total;
            }
            const int P0 = P_first;
            int i = 0;
            bool ok = true;
            bool waited = !a.early;
            // with a fused append, the tiles holding the rows this launch writes wait until the
            // copy warp has written them: the loop below runs in two phases, up to the first such
            // tile of the chunk and from it, and stays free of a per-tile check
            int bound = ntiles;
            if (fused) bound = first_written_tile(sg, lt, n, kh, ntiles, Ts, a);
            for (;;) {
            for (; i < bound; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait_bounded(empty0 + 8 * s, ((i / NS) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const Tile t = tile_at(sg, lt, pa);
                const bool deep = t.kind == kDeep;
                if (!waited && !deep) {  // ring rows: the previous launch may be writing the block
                    pdl_wait();
                    waited = true;
                }
                const int rows = deep ? pa.deep_box : pa.ring_box;
                const CUtensorMap *mk = deep ? &tmKd : &tmKw;
                const CUtensorMap *mv = deep ? &tmVd : &tmVw;
                const int z = deep ? ((a.layer * N + n) * kvH + kh)
                                   : (((a.layer * N + n) * a.R + t.plane) * kvH + kh);
                if constexpr (kDebug) {  // the tile lies inside its region and inside the plan
                    const bool bad =
                        t.cnt < 1 || t.cnt > rows ||
                        (deep ? (t.t0 < 0 || t.t0 + t.cnt > sg.D || sg.D > a.dbg_deep_rows || z >= a.dbg_deep_pages)
                              : (t.y < 0 || t.y + t.cnt > pa.ring_slots || t.t0 < sg.D ||
                                 t.t0 + t.cnt > (t.kind == kDual ? sg.T : sg.T + a.B) || z >= a.dbg_ring_pages ||
                                 (t.y - (t.t0 % pa.ring_slots) + pa.ring_slots) % pa.ring_slots != 0));
                    if (bad) atomicOr(a.err, RIPE_DEVERR_BOUNDS);
                }
                TileDesc &dsc = sdesc[s];
                dsc.pair = n * kvH + kh; dsc.n = n; dsc.kh = kh; dsc.T = sg.T;
                dsc.kind = t.kind; dsc.t0 = t.t0; dsc.cnt = t.cnt; dsc.plane = t.plane;
                const uint32_t fb = full0 + 8 * s;
                mbar_expect_tx(fb, 2 * C::NBOX * rows * 64);
                const uint32_t kdst = stage0 + s * C::STAGE_BYTES;
                const uint32_t vdst = kdst + C::NBOX * kBoxBytes;
#pragma unroll
                for (int b = 0; b < C::NBOX; ++b) {
                    tma_load_3d(kdst + b * kBoxBytes, mk, fb, b * kBoxCols, t.y, z);
                    tma_load_3d(vdst + b * kBoxBytes, mv, fb, b * kBoxCols, t.y, z);
                }
                if (++lt == sg.total) {
                    lt = 0;
                    if (++kh == kvH) {
                        kh = 0;
                        if (++n < N) sg = seq_geom(Ts[n], pa);
                    }
                }
                if (i == NS - 1) {  // pipeline full: warm L2 with the query rows of the later pairs
                    const int p_last = P_last;
                    for (int p = P0 + 1; p <= p_last; ++p) {
                        const int pn = p / kvH, pk = p - pn * kvH;
                        for (int j = 0; j < a.qB; ++j) {
                            const char *row = reinterpret_cast<const char *>(
                                a.q + ((static_cast<size_t>(pn) * a.qB + j) * a.Hq + pk * a.g) * D);
                            for (int off = 0; off < a.g * D * 2; off += 128)
                                asm volatile("prefetch.global.L2 [%0];" ::"l"(row + off));
                        }
                    }
                }
            }
            if (!ok || bound >= ntiles) break;
            // the copy warp wrote the block's rows into the ring (generic proxy) and fenced them
            if (!mbar_wait_bounded(smem_addr(&bars[2 * NS]), 0)) {
                ok = false;
                break;
            }
            bound = ntiles;
            }
            if (!ok) {
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                // drain: the last issue of every stage must land before the CTA exits
                for (int k = (i > NS ? i - NS : 0); k < i; ++k)
                    mbar_wait_bounded(full0 + 8 * (k % NS), (k / NS) & 1);
            }
        }
        return;  // the producer warp takes part in no consumer barrier (id 1)
    }
    if constexpr (C::SPLIT) setmaxnreg_inc<C::REG_CONSUMER>();


    // ==================================================================== consumers
    const int tg = warp / C::GW;             // tile group: tiles i with i % TG == tg
    const int rg = (warp % C::GW) / WK;      // row group: queries NQ*rg .. NQ*rg + NQ-1
    const int kg = warp % WK;                // key group: sub-blocks kg*SB .. kg*SB + SB-1
    const int g4 = lane >> 2, c4 = lane & 3;
    const int nct = C::NCW * 32;

    // query columns held by this thread: q = NQ*rg + 8*nq + 2*c4 + e  (e = 0, 1)
    int jq[NQT][2], lq[NQT][2];  // block position and loop of each query column held
    bool qvalid[NQT][2];
#pragma unroll
    for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int i = C::NQ * rg + 8 * nq + 2 * c4 + e;
            qvalid[nq][e] = i < a.Mq;
            jq[nq][e] = qvalid[nq][e] ? a.j0 + i / a.g : a.B - 1;
            lq[nq][e] = qvalid[nq][e] ? pa.jloop[jq[nq][e]] : -1;
        }
    // ldmatrix lane geometry (64-byte swizzle: 16-byte chunk ^= (row >> 1) & 3)
    const int mi = lane >> 3, r8 = lane & 7;
    const uint32_t swz = static_cast<uint32_t>(r8 >> 1);
    const uint32_t krow_off = static_cast<uint32_t>((mi & 1) * 8 + r8);  // K as A: (keys lo|hi) x (d lo|hi)
    const uint32_t kcol_sel = static_cast<uint32_t>(mi >> 1);
    const uint32_t vrow_off = static_cast<uint32_t>((mi >> 1) * 8 + r8); // V^T as A: (dv lo|hi) x (keys lo|hi)
    const uint32_t vcol_sel = static_cast<uint32_t>(mi & 1);

    float o[D / 16][NQT][4];
    // l_run sums the fp32 probabilities (the log-sum-exp); l_bf sums them as rounded to bf16 for
    // the P V product, so that the output is a true weighted average of V with those weights
    float m_ref[NQT][2], l_run[NQT][2], l_bf[NQT][2];
    uint32_t qb[D / 16][NQT][2];

    int fin_next = P_first;  // next pair to finalize (every consumer warp finalizes each pair once)
    int st_pair = -1;        // pair whose partial state this warp holds
    bool aborted = false;

    auto reset_state = [&]() {
#pragma unroll
        for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq) o[mt][nq][0] = o[mt][nq][1] = o[mt][nq][2] = o[mt][nq][3] = 0.f;
#pragma unroll
        for (int nq = 0; nq < NQT; ++nq) {
            m_ref[nq][0] = m_ref[nq][1] = -INFINITY;
            l_run[nq][0] = l_run[nq][1] = 0.f;
            l_bf[nq][0] = l_bf[nq][1] = 0.f;
        }
    };

    auto load_q = [&](int n, int kh) {
#pragma unroll
        for (int nq = 0; nq < NQT; ++nq) {
            const int i = C::NQ * rg + 8 * nq + g4;  // B-operand column = query g4 of the tile
            const uint32_t *qp = nullptr;
            if (i < a.Mq) {
                const int j = i / a.g, hg = i - j * a.g;
                qp = reinterpret_cast<const uint32_t *>(
                    a.q + ((static_cast<size_t>(n) * a.qB + j) * a.Hq + kh * a.g + hg) * D);
            }
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qb[ks][nq][0] = qp ? __ldg(qp + 8 * ks + c4) : 0u;
                qb[ks][nq][1] = qp ? __ldg(qp + 8 * ks + 4 + c4) : 0u;
            }
        }
    };

    // the CTAs holding tiles of pair p: c_first .. c_first + nparts - 1 (returns nparts)
    auto parts_of = [&](int p, int &c_first) -> int {
        const int n = p / kvH, kh = p - (p / kvH) * kvH;
        const int tot_n = (cum[n + 1] - cum[n]) / kvH;
        if (pieces) {
            c_first = p * pieces;
            return cdiv(tot_n, chunk);
        }
        const int start = cum[n] + kh * tot_n;
        c_first = start / chunk;
        return (start + tot_n - 1) / chunk - c_first + 1;
    };

    // ---------------------------------------------------------------- finalize one pair
    auto finalize = [&](int p, bool have) {
        const int n = p / kvH, kh = p - (p / kvH) * kvH;
        float *mw = mo + warp * C::NQ * C::DP;
        if (have) {
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float l = l_run[nq][e], lb = l_bf[nq][e];
                    l += __shfl_xor_sync(0xffffffffu, l, 4);
                    l += __shfl_xor_sync(0xffffffffu, l, 8);
                    l += __shfl_xor_sync(0xffffffffu, l, 16);
                    lb += __shfl_xor_sync(0xffffffffu, lb, 4);
                    lb += __shfl_xor_sync(0xffffffffu, lb, 8);
                    lb += __shfl_xor_sync(0xffffffffu, lb, 16);
                    l_run[nq][e] = l;
                    l_bf[nq][e] = lb;
                }
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt)
#pragma unroll
                for (int nq = 0; nq < NQT; ++nq) {
                    const int q0 = 8 * nq + 2 * c4;
                    mw[q0 * C::DP + 16 * mt + g4] = o[mt][nq][0];
                    mw[(q0 + 1) * C::DP + 16 * mt + g4] = o[mt][nq][1];
                    mw[q0 * C::DP + 16 * mt + 8 + g4] = o[mt][nq][2];
                    mw[(q0 + 1) * C::DP + 16 * mt + 8 + g4] = o[mt][nq][3];
                }
            if (g4 == 0) {
#pragma unroll
                for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int q = 8 * nq + 2 * c4 + e;
                        *reinterpret_cast<float4 *>(&mml[(warp * C::NQ + q) * 4]) =
                            make_float4(m_ref[nq][e], l_bf[nq][e], l_run[nq][e], 0.f);
                    }
            }
        } else {
            for (int q = lane; q < C::NQ; q += 32)
                *reinterpret_cast<float4 *>(&mml[(warp * C::NQ + q) * 4]) = make_float4(-INFINITY, 0.f, 0.f, 0.f);
        }
        named_bar_sync(1, nct);
        const bool abort_now = *reinterpret_cast<volatile int *>(&sflag[1]) != 0;
        int c_first;
        const int nparts = parts_of(p, c_first);
        const bool sole = nparts == 1;
        // per query row: the maximum over the warps that saw it, their weights and the sum
        for (int i = tid; i < C::ROWS; i += nct) {
            const int rgi = i / C::NQ, q = i - rgi * C::NQ;
            float M = -INFINITY;
#pragma unroll
            for (int t2 = 0; t2 < TG; ++t2)
#pragma unroll
                for (int k = 0; k < WK; ++k) M = fmaxf(M, mml[((t2 * C::GW + rgi * WK + k) * C::NQ + q) * 4]);
            float L = 0.f, Ll = 0.f;
#pragma unroll
            for (int t2 = 0; t2 < TG; ++t2)
#pragma unroll
                for (int k = 0; k < WK; ++k) {
                    const int w = t2 * C::GW + rgi * WK + k;
                    const float4 ml = *reinterpret_cast<const float4 *>(&mml[(w * C::NQ + q) * 4]);
                    const float f = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - M);
                    wq[i * (TG * WK) + t2 * WK + k] = f;
                    L += f * ml.y;
                    Ll += f * ml.z;
                }
            *reinterpret_cast<float4 *>(&fin[i * 4]) = make_float4(M, L, Ll, 0.f);
        }
        named_bar_sync(1, nct);
        // four consecutive columns of one row per thread: float4 shared-memory reads (the
        // row's weights are read once), 16-byte stores
        auto row_acc = [&](int i, int c0) {
            const int rgi = i / C::NQ, q = i - rgi * C::NQ;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int t2 = 0; t2 < TG; ++t2)
#pragma unroll
                for (int k = 0; k < WK; ++k) {
                    const float w = wq[i * (TG * WK) + t2 * WK + k];
                    if (w != 0.f) {
                        const float4 v = *reinterpret_cast<const float4 *>(
                            &mo[((t2 * C::GW + rgi * WK + k) * C::NQ + q) * C::DP + c0]);
                        acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
                    }
                }
            return acc;
        };
        constexpr int D4 = D / 4;
        if (C::XPAIR && a.xpair && pieces == 2 && !sole) {
            // a pair of CTAs holds this (sequence, kv head): the second sends its partial into
            // the first's shared memory, the first merges both and writes out / lse
            const uint32_t xbar = smem_addr(&bars[2 * NS + 1]);
            if (blockIdx.x & 1) {
                // asynchronous stores that complete the partner's expected byte count (sent even
                // after an abort, so that the partner never waits out its bound)
                const uint32_t rxo = mapa_shared(smem_addr(xo), 0), rxml = mapa_shared(smem_addr(xml), 0);
                const uint32_t rbar = mapa_shared(xbar, 0);
                for (int e = tid; e < a.Mq * D4; e += nct) {
                    const int i = e / D4, c0 = 4 * (e - i * D4);
                    const float4 acc = row_acc(i, c0);
                    st_async_v4(rxo + 4u * static_cast<uint32_t>(i * D + c0), acc, rbar);
                    if (c0 == 0)
                        st_async_v4(rxml + 16u * static_cast<uint32_t>(i), *reinterpret_cast<const float4 *>(&fin[i * 4]),
                                    rbar);
                }
            } else {
                // bounded wait for the partner's bytes
                const bool got = mbar_wait_cluster_bounded(xbar, 0);
                if (!got && tid == 0) atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                for (int e = tid; e < a.Mq * D4 && got && !abort_now; e += nct) {
                    const int i = e / D4, c0 = 4 * (e - i * D4);
                    const float4 acc = row_acc(i, c0);
                    const float4 o1 = *reinterpret_cast<const float4 *>(&xo[i * D + c0]);
                    const float4 f0 = *reinterpret_cast<const float4 *>(&fin[i * 4]);
                    const float4 f1 = *reinterpret_cast<const float4 *>(&xml[i * 4]);
                    const float M = fmaxf(f0.x, f1.x);
                    const float w0 = (f0.x == -INFINITY) ? 0.f : exp2f(f0.x - M);
                    const float w1 = (f1.x == -INFINITY) ? 0.f : exp2f(f1.x - M);
                    const float L = w0 * f0.y + w1 * f1.y, Ll = w0 * f0.z + w1 * f1.z;
                    const float inv = 1.f / L;
                    const int j = i / a.g, h = kh * a.g + (i - j * a.g);
                    const size_t orow = (static_cast<size_t>(n) * a.qB + j) * a.Hq + h;
                    __nv_bfloat162 *op = reinterpret_cast<__nv_bfloat162 *>(&a.out[orow * D + c0]);
                    op[0] = __floats2bfloat162_rn((w0 * acc.x + w1 * o1.x) * inv, (w0 * acc.y + w1 * o1.y) * inv);
                    op[1] = __floats2bfloat162_rn((w0 * acc.z + w1 * o1.z) * inv, (w0 * acc.w + w1 * o1.w) * inv);
                    if (c0 == 0 && a.lse) a.lse[orow] = (M + __log2f(Ll)) * 0.69314718055994531f;
                }
                named_bar_sync(1, nct);
            }
            return;
        }
        const int rows = sole ? a.Mq : C::ROWS;
        for (int e = tid; e < rows * D4 && !abort_now; e += nct) {
            const int i = e / D4, c0 = 4 * (e - i * D4);
            const float4 acc = row_acc(i, c0);  // a warp that saw no key of the row has weight 0
            if (sole) {
                const float inv = 1.f / fin[i * 4 + 1];
                const int j = i / a.g, h = kh * a.g + (i - j * a.g);
                const size_t orow = (static_cast<size_t>(n) * a.qB + j) * a.Hq + h;
                __nv_bfloat162 *op = reinterpret_cast<__nv_bfloat162 *>(&a.out[orow * D + c0]);
                op[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
                op[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
                if (c0 == 0 && a.lse) a.lse[orow] = (fin[i * 4] + __log2f(fin[i * 4 + 2])) * 0.69314718055994531f;
            } else {
                if (kDebug && static_cast<int>(blockIdx.x) + p >= a.dbg_part_slots) {
                    atomicOr(a.err, RIPE_DEVERR_BOUNDS);
                    continue;
                }
                const size_t prow = (static_cast<size_t>(blockIdx.x) + p) * C::ROWS + i;
                *reinterpret_cast<float4 *>(&a.part_o[prow * D + c0]) = acc;
                if (c0 == 0) *reinterpret_cast<float4 *>(&a.part_ml[prow * 4]) = *reinterpret_cast<const float4 *>(&fin[i * 4]);
            }
        }
        named_bar_sync(1, nct);  // partials written; the merge buffer is free again
        if (!sole && !abort_now && tid == 0) {
            // publish this CTA's partial (bar.sync + one fence covers every thread's writes)
            __threadfence();
            if (arrive_last(&a.counters[p], nparts, a.epoch)) {
                __threadfence();
                sflag[4 + sflag[3]] = p;  // merged at the end of this CTA's tiles
                sflag[3] += 1;
            }
        }
    };

    // ---------------------------------------------------------------- merge the partials of one pair
    // Runs in the CTA that arrived last, after all of its own tiles (the stage buffers are free).
    auto merge_pair = [&](int p) {
        const int n = p / kvH, kh = p - (p / kvH) * kvH;
        int c_first;
        const int nparts = parts_of(p, c_first);
        float *pw = reinterpret_cast<float *>(stages);  // [nparts][ROWS] m, then weights
        float *pl = pw + nparts * C::ROWS;              // [nparts][ROWS] l
        float *rowML = fin;                             // [ROWS][4] final M, L_out, L_lse
        for (int e = tid; e < nparts * a.Mq; e += nct) {
            const int c = e / a.Mq, i = e - (e / a.Mq) * a.Mq;
            const size_t prow = (static_cast<size_t>(c_first + c) + p) * C::ROWS + i;
            const float2 ml = __ldcg(reinterpret_cast<const float2 *>(&a.part_ml[prow * 4]));
            pw[c * C::ROWS + i] = ml.x;
            pl[c * C::ROWS + i] = ml.y;
        }
        named_bar_sync(1, nct);
        for (int i = tid; i < a.Mq; i += nct) {
            float M = -INFINITY;
            for (int c = 0; c < nparts; ++c) M = fmaxf(M, pw[c * C::ROWS + i]);
            float L = 0.f, Ll = 0.f;
            for (int c = 0; c < nparts; ++c) {
                const float mk = pw[c * C::ROWS + i];
                const float w = (mk == -INFINITY) ? 0.f : exp2f(mk - M);
                pw[c * C::ROWS + i] = w;
                L += w * pl[c * C::ROWS + i];
                const size_t prow = (static_cast<size_t>(c_first + c) + p) * C::ROWS + i;
                Ll += w * __ldcg(&a.part_ml[prow * 4 + 2]);
            }
            rowML[i * 4] = M;
            rowML[i * 4 + 1] = L;
            rowML[i * 4 + 2] = Ll;
        }
        named_bar_sync(1, nct);
        for (int e = tid; e < a.Mq * (D / 4); e += nct) {
            const int i = e / (D / 4), c4x = e - (e / (D / 4)) * (D / 4);
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
            for (int c = 0; c < nparts; ++c) {
                const float w = pw[c * C::ROWS + i];
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                    &a.part_o[((static_cast<size_t>(c_first + c) + p) * C::ROWS + i) * D + 4 * c4x]));
                acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
            }
            const float invL = 1.f / rowML[i * 4 + 1];
            const int j = i / a.g, h = kh * a.g + (i - j * a.g);
            const size_t orow = (static_cast<size_t>(n) * a.qB + j) * a.Hq + h;
            __nv_bfloat162 *op = reinterpret_cast<__nv_bfloat162 *>(&a.out[orow * D + 4 * c4x]);
            op[0] = __floats2bfloat162_rn(acc.x * invL, acc.y * invL);
            op[1] = __floats2bfloat162_rn(acc.z * invL, acc.w * invL);
            if (c4x == 0 && a.lse)
                a.lse[orow] = (rowML[i * 4] + __log2f(rowML[i * 4 + 2])) * 0.69314718055994531f;
        }
        if (tid == 0) a.counters[p] = 0;
        named_bar_sync(1, nct);
    };

    // ---------------------------------------------------------------- one tile
    auto compute = [&](const TileDesc &dsc, int s, auto fast_tag) {
        constexpr bool FAST = decltype(fast_tag)::value;
        const uint32_t kbase = stage0 + s * C::STAGE_BYTES;
        const uint32_t vbase = kbase + C::NBOX * kBoxBytes;
        float x[C::SB][NQT][4];
        bool act[C::SB];
#pragma unroll
        for (int sb = 0; sb < C::SB; ++sb) {
            const int kb = kg * C::SB + sb;
            act[sb] = FAST || 16 * kb < dsc.cnt;
            float se[NQT][4], so[NQT][4];
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
                for (int e = 0; e < 4; ++e) se[nq][e] = so[nq][e] = 0.f;
            if (act[sb]) {
                const uint32_t krow = static_cast<uint32_t>(16 * kb) + krow_off;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t col16 = static_cast<uint32_t>(2 * (ks & 1)) + kcol_sel;
                    const uint32_t addr = kbase + (ks >> 1) * kBoxBytes + krow * 64 + ((col16 ^ swz) << 4);
                    uint32_t af[4];
                    ldsm_x4(addr, af[0], af[1], af[2], af[3]);
#pragma unroll
                    for (int nq = 0; nq < NQT; ++nq) {
                        if (ks & 1) mma_16816(so[nq], af, qb[ks][nq][0], qb[ks][nq][1]);
                        else mma_16816(se[nq], af, qb[ks][nq][0], qb[ks][nq][1]);
                    }
                }
            }
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v = (se[nq][e] + so[nq][e]) * a.scale_log2;
                    if (!FAST) {
                        const int kk = 16 * kb + g4 + 8 * (e >> 1);
                        const int tpos = dsc.t0 + kk;
                        const int pq = dsc.T + jq[nq][e & 1];
                        bool vis = act[sb] && kk < dsc.cnt;
                        if (dsc.kind == kRing)  // the ring at plane r serves only the queries of loop r
                            vis = vis && lq[nq][e & 1] == dsc.plane && tpos <= pq &&
                                  (pa.mode_eff != 0 || tpos >= dsc.T || tpos >= pq - pa.W);
                        else if (dsc.kind == kDual)
                            vis = vis && tpos < pq - pa.W;
                        if constexpr (FUSED) {  // windowed draft: sink and sliding window only
                            if (pa.dwin >= 0) vis = vis && (tpos < pa.sink || tpos >= pq - pa.dwin);
                        }
                        v = vis ? v : -INFINITY;
                    }
                    x[sb][nq][e] = v;
                }
        }
        // column maxima over this thread's keys; the reference of a column moves only when its
        // maximum over the warp exceeds the reference by more than kLazyMax, which is so exactly
        // when one lane's own maximum does.  Only then are the maxima reduced over the 8 lanes
        // sharing a column (most tiles skip those shuffles, and their exponentials do not wait)
        float mloc[NQT][2];
        bool over = false;
#pragma unroll
        for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                float mt = -INFINITY;
#pragma unroll
                for (int sb = 0; sb < C::SB; ++sb) mt = fmaxf(mt, fmaxf(x[sb][nq][e], x[sb][nq][e + 2]));
                mloc[nq][e] = mt;
                over = over || mt > m_ref[nq][e] + kLazyMax;  // also true for a finite maximum when m_ref is -inf
            }
        if (__any_sync(0xffffffffu, over)) {
            float alpha[NQT][2];
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float mt = mloc[nq][e];
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
                    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
                    alpha[nq][e] = 1.f;
                    if (mt > m_ref[nq][e] + kLazyMax) {
                        alpha[nq][e] = exp2f(m_ref[nq][e] - mt);
                        m_ref[nq][e] = mt;
                    }
                }
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq) {
                l_run[nq][0] *= alpha[nq][0];
                l_run[nq][1] *= alpha[nq][1];
                l_bf[nq][0] *= alpha[nq][0];
                l_bf[nq][1] *= alpha[nq][1];
#pragma unroll
                for (int mt = 0; mt < D / 16; ++mt) {
                    o[mt][nq][0] *= alpha[nq][0]; o[mt][nq][1] *= alpha[nq][1];
                    o[mt][nq][2] *= alpha[nq][0]; o[mt][nq][3] *= alpha[nq][1];
                }
            }
        }
        // P^T fragments: rows (keys) g4 / g4+8, columns (queries) 2c4, 2c4+1 -> movmatrix
#pragma unroll
        for (int sb = 0; sb < C::SB; ++sb) {
            if (!act[sb]) continue;
            const int kb = kg * C::SB + sb;
            uint32_t pb[NQT][2];
#pragma unroll
            for (int nq = 0; nq < NQT; ++nq) {
                const float r0 = m_ref[nq][0], r1 = m_ref[nq][1];
                const float p0 = (r0 == -INFINITY) ? 0.f : exp2f(x[sb][nq][0] - r0);
                const float p1 = (r1 == -INFINITY) ? 0.f : exp2f(x[sb][nq][1] - r1);
                const float p2 = (r0 == -INFINITY) ? 0.f : exp2f(x[sb][nq][2] - r0);
                const float p3 = (r1 == -INFINITY) ? 0.f : exp2f(x[sb][nq][3] - r1);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(p0, p1);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(p2, p3);
                // two normalisers: the rounded probabilities the P V product sees (the output is
                // their weighted average of V) and the fp32 ones (the lse stays fp32-accurate)
                l_run[nq][0] += p0 + p2;
                l_run[nq][1] += p1 + p3;
                l_bf[nq][0] += __low2float(lo) + __low2float(hi);
                l_bf[nq][1] += __high2float(lo) + __high2float(hi);
                pb[nq][0] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&lo));
                pb[nq][1] = movmatrix_t(*reinterpret_cast<const uint32_t *>(&hi));
            }
            // O^T += V^T P^T
            const uint32_t vrow = static_cast<uint32_t>(16 * kb) + vrow_off;
#pragma unroll
            for (int mt = 0; mt < D / 16; ++mt) {
                const uint32_t col16 = static_cast<uint32_t>(2 * (mt & 1)) + vcol_sel;
                const uint32_t addr = vbase + (mt >> 1) * kBoxBytes + vrow * 64 + ((col16 ^ swz) << 4);
                uint32_t af[4];
                ldsm_x4_t(addr, af[0], af[1], af[2], af[3]);
#pragma unroll
                for (int nq = 0; nq < NQT; ++nq) mma_16816(o[mt][nq], af, pb[nq][0], pb[nq][1]);
            }
        }
    };

    // ring tiles can take the mask-free path only when every query is at the tile's loop and no
    // draft window cuts keys out
    const bool ring_all_visible = pa.nloops == 1 && pa.dwin < 0;
    reset_state();
    // the first pair's queries: loaded while its first tile is still in flight (with an early
    // start, once the previous launch has finished: the caller may be writing them)
    st_pair = P_first;
    if (a.early) pdl_wait();
    load_q(P_first / kvH, P_first - (P_first / kvH) * kvH);
    for (int i = tg; i < ntiles; i += TG) {
        const int s = i % NS;
        if (!mbar_wait_bounded(full0 + 8 * s, (i / NS) & 1)) {
            aborted = true;
            atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            break;
        }
        const TileDesc dsc = sdesc[s];
        if (dsc.pair != st_pair) {
            while (fin_next < dsc.pair) {
                finalize(fin_next, st_pair == fin_next);
                ++fin_next;
            }
            st_pair = dsc.pair;
            reset_state();
            load_q(dsc.n, dsc.kh);
        }
        // mask-free: a full deepest-plane tile, or a full ring tile that every query of the call
        // sees whole (one loop; every key before the first query and inside the last query's
        // window, as for the full cache and windows wider than the prefix)
        const bool full_view =
            dsc.cnt == kTileRows &&
            (dsc.kind == kDeep ||
             (dsc.kind == kRing && ring_all_visible && dsc.t0 + kTileRows - 1 <= dsc.T + a.j0 &&
              (pa.mode_eff != 0 || dsc.t0 >= dsc.T + a.j0 + a.qB - 1 - pa.W)));
        if (full_view)
            compute(dsc, s, std::integral_constant<bool, true>());
        else
            compute(dsc, s, std::integral_constant<bool, false>());
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
    }
    while (fin_next <= P_last) {
        finalize(fin_next, !aborted && st_pair == fin_next);
        ++fin_next;
    }
    named_bar_sync(1, nct);
    if (*reinterpret_cast<volatile int *>(&sflag[1]) == 0) {
        const int nm = sflag[3];
        for (int k = 0; k < nm; ++k) merge_pair(sflag[4 + k]);
    }
}

// ---------------------------------------------------------------- host side
// The per-function limit on dynamic shared memory.  A launch asks for smem_bytes_for<C>(N),
// which grows with the batch N (the per-sequence tile counts live in shared memory).  The
// limit is raised once per device to what the largest batch asks for, so that no cache
// allocation or call ever lowers it below what a live cache of a larger batch needs.
template <class C>
constexpr int kSmemMax = smem_bytes_for<C>(kMaxBatch);

template <int D, int NQT, int WR, int WK, int TG>
struct Inst {
    using C = VCfg<D, NQT, WR, WK, TG>;
    static_assert(kSmemMax<C> <= kSmemLimit, "the largest batch's shared memory must fit a CTA");
    static constexpr auto kernel = ripe_verify_kernel<D, NQT, WR, WK, TG, false>;
    static constexpr auto kernel_fused = ripe_verify_kernel<D, NQT, WR, WK, TG, true>;
    // The register split assumes the kernels are launched at LAUNCH_REGS per thread; with fewer, the
    // consumers' setmaxnreg.inc could never be satisfied: refuse the kernels instead.
    static cudaError_t check_registers() {
        if constexpr (C::SPLIT) {
            for (auto k : {kernel, kernel_fused}) {
                cudaFuncAttributes fa;
                const cudaError_t e = cudaFuncGetAttributes(&fa, k);
                if (e != cudaSuccess) return e;
                if (fa.numRegs * C::THREADS < C::NCW * 32 * C::REG_CONSUMER + 4 * 32 * C::REG_PRODUCER)
                    return cudaErrorInvalidConfiguration;
            }
        }
        return cudaSuccess;
    }
    static cudaError_t set_attr_max() {
        cudaError_t e = check_registers();
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax<C>);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kernel_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemMax<C>);
        return e;
    }
    // 2 x the clusters of two CTAs that fit at once (0: no cluster launch), per device, instance
    // and shared-memory size
    static int pair_grid(bool fused, int smem, int device, int num_sms) {
        struct Entry {
            int smem = -1, grid = 0;
        };
        static Entry cache[kMaxDevices][2];
        static std::mutex mu;
        const int f = fused ? 1 : 0;
        std::lock_guard<std::mutex> lock(mu);
        Entry &e = cache[device][f];
        if (e.smem != smem) {
            const int n = max_active_clusters(fused ? kernel_fused : kernel, dim3(C::threads(fused)), smem, 2,
                                              num_sms & ~1);
            e.grid = 2 * n;
            e.smem = smem;
        }
        return e.grid;
    }
    static cudaError_t launch(const LaunchTarget &t, int grid, const VerifyArgs &args, cudaStream_t s) {
        if (grid > C::MAX_PARTS) grid = C::MAX_PARTS;
        const bool fused = args.blk_k != nullptr;
        auto kern = fused ? kernel_fused : kernel;
        const dim3 block(C::threads(fused));
        const int smem = smem_bytes_for<C>(t.N);
        VerifyArgs a = args;
        a.xpair = 0;
#ifndef RIPE_NO_XPAIR
        if (C::XPAIR) {
            const int pg = pair_grid(fused, smem, t.device, t.num_sms);
            if (pg >= 2) {
                int g2 = (grid + 1) & ~1;
                if (g2 > pg) g2 = pg;
                a.xpair = 1;
                return launch_pdl_cluster(kern, dim3(g2), block, smem, s, 2, *t.tmKd, *t.tmVd, *t.tmKw, *t.tmVw, a);
            }
        }
#endif
        return launch_pdl(kern, dim3(grid), block, smem, s, *t.tmKd, *t.tmVd, *t.tmKw, *t.tmVw, a);
    }
};

// query-side configuration by the number of query rows per kv head (B * group)
//   <= 8  : one 8-query tile per warp, 2 tile groups of 4 warps
//   <= 16 : two 8-query tiles per warp, 2 tile groups of 4 warps
//   <= 32 : two row groups x 2 key groups, 2 tile groups (measured on the long-context GQA call:
//           181 us vs 196-199 us for one tile group of 2 x 4 warps, whose 32 KB stages fit only 3 deep)
//   <= 64 : four row groups x 2 key groups (32 keys per warp per tile)
#ifndef RIPE_Q8_WK
#define RIPE_Q8_WK 4
#define RIPE_Q8_TG 2
#endif
#ifndef RIPE_Q32_NQT
#define RIPE_Q32_NQT 2
#define RIPE_Q32_WR 2
#define RIPE_Q32_WK 2
#define RIPE_Q32_TG 2
#endif
#define RIPE_Q32_CFG RIPE_Q32_NQT, RIPE_Q32_WR, RIPE_Q32_WK, RIPE_Q32_TG
#define RIPE_QCFG_LIST(D)                                                          \
    Inst<D, 1, 1, RIPE_Q8_WK, RIPE_Q8_TG>, Inst<D, 2, 1, 4, 2>, Inst<D, RIPE_Q32_CFG>, Inst<D, 2, 4, 2, 1>

static int qcfg_of(int Mq) { return Mq <= 8 ? 0 : Mq <= 16 ? 1 : Mq <= 32 ? 2 : 3; }

template <class... I>
static cudaError_t set_all_max() {
    cudaError_t e = cudaSuccess;
    ((e = (e == cudaSuccess ? I::set_attr_max() : e)), ...);
    return e;
}

int ensure_verify_attributes(int device) {
    if (device < 0 || device >= kMaxDevices) return RIPE_EINVAL;
    static bool done[kMaxDevices] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (done[device]) return RIPE_OK;
    int cur = -1;
    if (cudaGetDevice(&cur) != cudaSuccess || cur != device) return RIPE_ECUDA;  // caller makes it current
    cudaError_t e = set_all_max<RIPE_QCFG_LIST(64)>();
    if (e == cudaSuccess) e = set_all_max<RIPE_QCFG_LIST(96)>();
    if (e == cudaSuccess) e = set_all_max<RIPE_QCFG_LIST(128)>();
    if (e == cudaSuccess) e = set_verify_tc_attributes();
    if (e != cudaSuccess) {
        cudaGetLastError();
        return RIPE_ECUDA;
    }
    done[device] = true;
    return RIPE_OK;
}

template <class I0, class I1, class I2, class I3>
static cudaError_t launch_d(int qc, const LaunchTarget &t, int grid, const VerifyArgs &a, cudaStream_t s) {
    switch (qc) {
        case 0: return I0::launch(t, grid, a, s);
        case 1: return I1::launch(t, grid, a, s);
        case 2: return I2::launch(t, grid, a, s);
        default: return I3::launch(t, grid, a, s);
    }
}

// The consumer for 9..64 query rows per kv head (ripe_set_verify_consumer).  By default this
// file's mma.sync kernel: on B200 it measured faster than the tcgen05 kernel (ripe_verify_tc.cu) at
// every shape tried (8 sequences x 8 kv heads, L2 flushed, per call: 64 rows, head_dim 128, 32K keys
// 283 vs 297 us; 4K keys 64 vs 76 us; head_dim 96 / 64 at 32K keys 265 vs 293 / 217 vs 266 us; 40
// rows 281 vs 316 us; 32 rows 193 vs 244 us; 16 rows 188 vs 246 us).  Launches that write the draft
// block (fused append, draft steps) always use this file's kernel.
static std::atomic<int> g_consumer{-1};  // -1: not read from the environment yet

static int consumer_choice() {
    int c = g_consumer.load(std::memory_order_relaxed);
    if (c < 0) {
        const char *e = std::getenv("RIPE_VERIFY_CONSUMER");
        const int env = (e && std::strcmp(e, "mma") == 0) ? RIPE_CONSUMER_MMA
                        : (e && std::strcmp(e, "tc") == 0) ? RIPE_CONSUMER_TC
                                                           : RIPE_CONSUMER_DEFAULT;
        int expected = -1;
        g_consumer.compare_exchange_strong(expected, env);
        c = g_consumer.load(std::memory_order_relaxed);
    }
    return c;
}

int get_verify_consumer() { return consumer_choice(); }

int set_verify_consumer(int consumer) {
    if (consumer < RIPE_CONSUMER_DEFAULT || consumer > RIPE_CONSUMER_TC) return RIPE_EINVAL;
    const int prev = consumer_choice();
    g_consumer.store(consumer, std::memory_order_relaxed);
    return prev;
}

// tiles: the launch's 64-key tiles when known on the host, else -1
static cudaError_t launch_any(int d, int qc, const LaunchTarget &t, int grid, const VerifyArgs &a,
                              cudaStream_t s) {
    if (qc >= 1 && a.blk_k == nullptr && consumer_choice() == RIPE_CONSUMER_TC)
        return launch_verify_tc(d, t, grid, a, s);
    switch (d) {
        case 64: return launch_d<RIPE_QCFG_LIST(64)>(qc, t, grid, a, s);
        case 96: return launch_d<RIPE_QCFG_LIST(96)>(qc, t, grid, a, s);
        case 128: return launch_d<RIPE_QCFG_LIST(128)>(qc, t, grid, a, s);
        default: return cudaErrorInvalidValue;
    }
}

int verify_rows_for(int Mq) { return 8 << qcfg_of(Mq); }

// Launch over explicitly given buffers and scratch (the allocation-free entry point).
int launch_verify_raw(const RawVerify &rv, cudaStream_t s) {
    VerifyArgs a;
    a.blk_k = a.blk_v = nullptr;
    a.ring_k = a.ring_v = nullptr;
    a.max_T = 0;
    a.xpair = 0;
    a.epoch = rv.epoch;
    a.q = static_cast<const __nv_bfloat16 *>(rv.q);
    a.out = static_cast<__nv_bfloat16 *>(rv.out);
    a.lse = rv.lse;
    a.T = rv.T;
    a.part_o = rv.part_o;
    a.part_ml = rv.part_ml;
    a.counters = rv.counters;
    a.err = rv.err;
    a.plan = rv.plan;
    a.N = rv.N;
    a.kvH = rv.kvH;
    a.g = rv.g;
    a.Hq = rv.Hq;
    a.B = rv.plan.B;
    a.j0 = 0;
    a.qB = rv.plan.B;
    a.R = rv.plan.R;
    a.layer = rv.layer;
    a.Mq = rv.plan.B * rv.g;
    a.min_chunk = RIPE_MIN_CHUNK;
    a.has_deep = rv.has_deep;
    a.dbg_deep_rows = rv.dbg_deep_rows;
    a.dbg_part_slots = rv.grid + rv.N * rv.kvH;
    a.dbg_deep_pages = rv.dbg_deep_pages;
    a.dbg_ring_pages = rv.dbg_ring_pages;
    a.early = 0;  // the caller's own kernels may write the cache buffers
    a.scale_log2 = rv.scale * 1.4426950408889634f;
    const LaunchTarget t = {&rv.tmKd, &rv.tmVd, &rv.tmKw, &rv.tmVw, rv.device, rv.num_sms, rv.N};
    if (rv.d != 64 && rv.d != 96 && rv.d != 128) return RIPE_EINVAL;
    return launch_any(rv.d, qcfg_of(a.Mq), t, rv.grid, a, s) == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}
static int launch_cache_args(ripe_cache *c, int layer, VerifyArgs &a, float scale, cudaStream_t s);

// One loop r; block positions [0, B) in the tile plan, queries at positions j0 .. j0 + qB - 1.
static int launch_single_loop(ripe_cache *c, int layer, int r, int B, int j0, int qB, const void *q, void *out,
                              float *lse, float scale, cudaStream_t s, const void *blk_k, const void *blk_v,
                              int sink = 0, int dwin = -1) {
    VerifyArgs a;
    a.epoch = 0;
    a.blk_k = static_cast<const uint4 *>(blk_k);
    a.blk_v = static_cast<const uint4 *>(blk_v);
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.j0 = j0;
    a.qB = qB;
    a.plan.W = c->W;
    a.plan.B = B;
    a.plan.R = c->R;
    a.plan.sink = sink;
    a.plan.dwin = dwin;
    a.plan.dj = j0;
    a.plan.ring_slots = c->ring_slots;
    a.plan.deep_box = c->deep_box;
    a.plan.ring_box = c->ring_box;
    // at the deepest loop every key reads plane R-1, so the window rule changes nothing
    a.plan.mode_eff = (c->mode == RIPE_WINDOW_CACHE_RELATIVE || r == c->R - 1) ? 1 : 0;
    a.plan.nloops = 1;
    a.plan.loop[0] = static_cast<uint8_t>(r);
    for (int j = 0; j < kMaxQueryRows; ++j) a.plan.jloop[j] = static_cast<uint8_t>(r);
    return launch_cache_args(c, layer, a, scale, s);
}

int launch_verify(ripe_cache *c, int layer, int r, const void *q, void *out, float *lse, float scale,
                  cudaStream_t s, const void *blk_k, const void *blk_v) {
    return launch_single_loop(c, layer, r, c->B_cur, 0, c->B_cur, q, out, lse, scale, s, blk_k, blk_v);
}

// Draft step: position j of the block at loop r, its K/V written by the same launch.
int launch_draft(ripe_cache *c, int layer, int r, int j, const void *k, const void *v, const void *q, void *out,
                 float *lse, float scale, cudaStream_t s, int sink, int window) {
    return launch_single_loop(c, layer, r, j + 1, j, 1, q, out, lse, scale, s, k, v, sink, window);
}

// Several loops in one call: block position j is verified at loop loop_of_position[j].
int launch_verify_wave(ripe_cache *c, int layer, const int32_t *loop_of_position, const void *q, void *out,
                       float *lse, float scale, cudaStream_t s) {
    VerifyArgs a;
    a.epoch = 0;
    a.blk_k = a.blk_v = nullptr;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.j0 = 0;
    a.qB = c->B_cur;
    a.plan.W = c->W;
    a.plan.B = c->B_cur;
    a.plan.R = c->R;
    a.plan.sink = 0;
    a.plan.dwin = -1;
    a.plan.dj = 0;
    a.plan.ring_slots = c->ring_slots;
    a.plan.deep_box = c->deep_box;
    a.plan.ring_box = c->ring_box;
    a.plan.mode_eff = c->mode == RIPE_WINDOW_CACHE_RELATIVE ? 1 : 0;
    bool used[kMaxLoops] = {false};
    for (int j = 0; j < c->B_cur; ++j) used[loop_of_position[j]] = true;
    a.plan.nloops = 0;
    for (int r = 0; r < c->R; ++r)
        if (used[r]) a.plan.loop[a.plan.nloops++] = static_cast<uint8_t>(r);
    for (int j = 0; j < kMaxQueryRows; ++j)
        a.plan.jloop[j] = static_cast<uint8_t>(j < c->B_cur ? loop_of_position[j] : loop_of_position[0]);
    return launch_cache_args(c, layer, a, scale, s);
}

static int launch_cache_args(ripe_cache *c, int layer, VerifyArgs &a, float scale, cudaStream_t s) {
    a.ring_k = reinterpret_cast<uint4 *>(c->Kw);
    a.ring_v = reinterpret_cast<uint4 *>(c->Vw);
    a.max_T = c->max_T;
    a.T = c->T_dev;
    a.part_o = c->part_o;
    a.part_ml = c->part_ml;
    a.counters = c->counters;
    a.err = c->err_dev;
    a.N = c->N;
    a.kvH = c->kvH;
    a.g = c->g;
    a.Hq = c->Hq;
    a.B = a.plan.B;
    a.R = c->R;
    a.layer = layer;
    a.Mq = a.qB * c->g;
    a.min_chunk = RIPE_MIN_CHUNK;  // bounds the number of partials of one (sequence, kv head)
    a.has_deep = c->deep_rows > 0 ? 1 : 0;
    a.dbg_deep_rows = c->deep_rows;
    a.dbg_part_slots = c->part_slots;
    a.dbg_deep_pages = static_cast<long long>(c->L) * c->N * c->kvH;
    a.dbg_ring_pages = static_cast<long long>(c->L) * c->N * c->R * c->kvH;
    a.early = c->lengths_dirty ? 0 : 1;
    a.scale_log2 = scale * 1.4426950408889634f;
    const int qc = qcfg_of(a.Mq);

    // grid: one CTA per SM, fewer when the host copy of T says there is less work
    int grid = c->num_sms < 256 ? c->num_sms : 256;  // the last-CTA merge keeps <= 256 partial weights per row
    if (c->synced) {
        long total = 0;
        for (int n = 0; n < c->N; ++n) total += static_cast<long>(seq_geom(c->T[n], a.plan).total) * c->kvH;
        const long need = (total + a.min_chunk - 1) / a.min_chunk;
        if (need < grid) grid = static_cast<int>(need);
    }
    if (grid < 1) grid = 1;
    if (c->d != 64 && c->d != 96 && c->d != 128) return RIPE_EINVAL;
    const LaunchTarget t = {&c->tm_Kd, &c->tm_Vd, &c->tm_Kw, &c->tm_Vw, c->device, c->num_sms, c->N};
    const cudaError_t e = launch_any(c->d, qc, t, grid, a, s);
    c->launches += 1;
    c->lengths_dirty = false;
    return e == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

}  // namespace ripe
