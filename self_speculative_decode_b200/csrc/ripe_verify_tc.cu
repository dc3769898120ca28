// Verification attention over a RIPE multi-plane KV cache with the fifth-generation tensor
// cores (tcgen05, accumulators in tensor memory), for 9..64 query rows per kv head (sm_100a).
//
// What is computed is exactly what ripe_verify.cu computes (RIPE abstract, "Prefix Keys and
// Values Matter Late: RIPE Caching for Self-Speculative Decoding in Looped Language Models",
// first, fourth and fifth sentences): for every query of the draft block at loop r, causal softmax
// attention over the keys t <= p, each read at plane r (draft block, window) or at the deepest
// plane R-1.  The tile plan, the chunking of the tile lists over CTAs, the early start and the
// last-arrival merge of split partials are shared with that kernel; only the consumer differs.
//
// Roles (192 threads):
//   warps 0-3  softmax / epilogue.  The MMA's M = 64 rows sit in tensor-memory lanes
//              32 w + (0..15) of quadrant w, and only warp w (sub-partition w) may read them.  The
//              query rows are spread over the quadrants first: rpq = 4, 8 or 16 rows per quadrant
//              (up to 16, 32 or 64 rows), query row w rpq + l in MMA row 16 w + l.
//   warp 4     producer: one thread streams 64-key tiles with 3-D TMA loads (no multicast) into
//              an NS-stage ring.  A stage's K and V halves have barriers of their own: K of tile
//              t is loaded KA tiles ahead of V of tile t, and the K half is reloaded as soon as
//              S of its tile is computed.
//   warp 5     MMA: allocates tensor memory; one thread issues, as each becomes ready,
//                S[i & 1] = Q K_i^T   (M = 64 query rows, N = 64 keys, K = head_dim)
//              once K_i has landed and the softmax has read S[i & 1] of tile i - 2, and
//                O += P_i V_i         (M = 64, N = head_dim, K = 64 keys; V read in place from the
//                                      TMA stage as an MN-major operand)
//              once the softmax has written P_i (bf16, shared memory) and V_i has landed; each
//              product frees its half of the stage with tcgen05.commit.
// The softmax takes one tile per iteration (two with RIPE_TC_PAIR) and keeps the row's running
// maximum m and sums l in registers (base 2).  The maximum moves only when a tile's maximum
// exceeds it by more than 8 (exact; the rescale of O, a tensor-memory read-modify-write of the
// thread's row, is then rare).  Rows past the query count are zero in Q and never written out.
#include <mutex>
#include <type_traits>

#include "ripe_verify.cuh"

#ifndef RIPE_TC_MAX_STAGES
#define RIPE_TC_MAX_STAGES 8  // K/V stage cap (shared memory sets the rest)
#endif
#ifndef RIPE_TC_PAIR
// 1: the softmax takes two tiles of a (sequence, kv head) per iteration; 0 (measured faster at 32
// and 64 query rows: 244 vs 254 us and 297 vs 305 us per long-context call): one
#define RIPE_TC_PAIR 0
#endif
#ifndef RIPE_TC_K_AHEAD
#define RIPE_TC_K_AHEAD 3     // tiles by which the K loads run ahead of the V loads
#endif

namespace ripe {

// ---------------------------------------------------------------- tcgen05 / TMEM wrappers
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// arrive once on an mbarrier when every tcgen05 operation this thread issued so far has completed
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// D (tensor memory) = A (shared) * B (shared) [+ D], bf16 inputs, fp32 accumulate
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Loads and stores of 16 tensor-memory lanes (the warp's lane quadrant, lanes 0-15: the rows of an
// M = 64 accumulator) x 256 bits per repetition.  Thread t holds lanes t / 4 and t / 4 + 8 at 32-bit
// columns 8 k + 2 (t % 4) + {0, 1}: register 4 k + 2 h + e is lane t / 4 + 8 h, column 8 k + 2 (t % 4) + e.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st_16x256b_x4(uint32_t taddr, const uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x4.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// non-blocking: has the phase with the given parity completed?
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// generic-proxy shared-memory writes -> visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Shared-memory matrix descriptor (sm_100 format, version 1) of a 64-byte-swizzled operand.
//   K-major (rows contiguous along K): 8-row groups 512 B apart (SBO); LBO unused (16 B)
//   MN-major (rows contiguous along M/N): 8-row K groups 512 B apart (SBO), 32-wide M/N groups
//   one 4 KB box apart (LBO)
__device__ __forceinline__ uint64_t sw64_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    return static_cast<uint64_t>((addr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (4ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, fp32 D, M = 64, N, A K-major, B K- or MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_m64(int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(64 >> 4) << 24);
}

// query rows per partial slot of the merge scratch: 8, 16, 32 or 64 (as for the mma.sync kernel)
__device__ __forceinline__ int part_rows(int Mq) { return Mq <= 8 ? 8 : Mq <= 16 ? 16 : Mq <= 32 ? 32 : 64; }

// ---------------------------------------------------------------- configuration
template <int D>
struct TcCfg {
    static constexpr int NBOX = D / kBoxCols;                // 64-byte column boxes per row
    static constexpr int STAGE_BYTES = 2 * NBOX * kBoxBytes; // K and V of one 64-key tile
    static constexpr int Q_BYTES = NBOX * kBoxBytes;         // 64 query rows
    static constexpr int P_BYTES = 2 * kBoxBytes;            // 64 rows x 64 keys, bf16
    static constexpr int MROWS = 64;                         // the MMA's M (query rows, padded)
    static constexpr int NSW = 4;                            // softmax warps
    static constexpr int PRODUCER = 4, MMA_WARP = 5;
    static constexpr int THREADS = 6 * 32;
    static constexpr int TMEM_COLS = 256;                    // S[0], S[1] (64 columns each), O (D columns)
    static constexpr int S_COL = 0, O_COL = 128;
    static constexpr int FIN_BYTES = MROWS * 4 * 4;          // per-row (M, L_out, L_lse) of a merge
    static constexpr int MISC = 1024 /*align*/ + 1024 /*bars, descriptors, flags*/;
    static constexpr int NPB = 4;                            // P buffers
    static constexpr int FIXED = MISC + Q_BYTES + NPB * P_BYTES + FIN_BYTES;
    static constexpr int AVAIL = kSmemLimit - FIXED - 4 * (2 * kMaxBatch + 2);
    static constexpr int NS = AVAIL / STAGE_BYTES > RIPE_TC_MAX_STAGES ? RIPE_TC_MAX_STAGES : AVAIL / STAGE_BYTES;
    static constexpr int KA = NS - 1 < RIPE_TC_K_AHEAD ? NS - 1 : RIPE_TC_K_AHEAD;
    static_assert(NS >= 3, "not enough shared memory for the pipeline");
    static constexpr int SMEM_FIXED = FIXED + NS * STAGE_BYTES;
    static_assert(SMEM_FIXED + 4 * (2 * kMaxBatch + 2) <= kSmemLimit, "shared memory");
    // the end-of-CTA merge keeps (m, l) of up to MAX_PARTS partials x 64 rows in the stage, Q and P
    // buffers (contiguous, all free by then): at most MAX_PARTS CTAs (enough for a 148-SM B200)
    static constexpr int MERGE_BYTES = NS * STAGE_BYTES + Q_BYTES + NPB * P_BYTES;
    static constexpr int MAX_PARTS = MERGE_BYTES / (MROWS * 2 * 4) < 256 ? MERGE_BYTES / (MROWS * 2 * 4) : 256;
    static_assert(MAX_PARTS >= 148, "stage buffers too small for the merge");
};

__host__ __device__ constexpr int tc_smem_bytes(int fixed, int N) { return fixed + (2 * N + 2) * 4; }

// ---------------------------------------------------------------- the kernel
template <int D>
__global__ void __launch_bounds__(TcCfg<D>::THREADS, 1)
ripe_verify_tc_kernel(const __grid_constant__ CUtensorMap tmKd, const __grid_constant__ CUtensorMap tmVd,
                      const __grid_constant__ CUtensorMap tmKw, const __grid_constant__ CUtensorMap tmVw,
                      const __grid_constant__ VerifyArgs a) {
    using C = TcCfg<D>;
    constexpr int NS = C::NS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stages = base;                                      // [NS][K | V]
    uint8_t *qs = stages + NS * C::STAGE_BYTES;                  // Q, K-major, 64-byte swizzle
    uint8_t *ps = qs + C::Q_BYTES;                               // P[NPB]
    float *fin = reinterpret_cast<float *>(ps + C::NPB * C::P_BYTES);  // [64][4] merge M, L_out, L_lse
    uint64_t *bars = reinterpret_cast<uint64_t *>(fin + C::MROWS * 4);
    // fullK[NS] fullV[NS] emptyK[NS] emptyV[NS] sfull[2] sfree[2] pfull[NPB] pvdone[NPB] qready mmadone esync
    TileDesc *sdesc = reinterpret_cast<TileDesc *>(bars + 4 * NS + 7 + 2 * C::NPB);  // [NS]
    int2 *vsrc = reinterpret_cast<int2 *>(sdesc + NS);                    // [NS] row and page of a tile's V
    int *sflag = reinterpret_cast<int *>(vsrc + NS);                      // [16]; sflag[8] = TMEM base
    int *cum = sflag + 16;                                                // [N + 1]
    int *Ts = cum + a.N + 1;                                              // [N]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;
    // query rows per tensor-memory lane quadrant: the rows are spread over all four quadrants, and so
    // over the four SM sub-partitions (a warp reads only the quadrant of its sub-partition), before
    // any quadrant takes more than 4 or 8
    const int rpq = a.Mq > 32 ? 16 : a.Mq > 16 ? 8 : 4;
    const int nsw = (a.Mq + rpq - 1) / rpq;  // softmax warps with rows
    const int nst = nsw * 32;          // their threads

    // a stage's K and V halves fill and drain separately: K is free once S = Q K^T is computed and
    // the softmax warps have read the tile's descriptor, V once the P V product is
    const uint32_t fullK0 = smem_addr(&bars[0]);
    const uint32_t fullV0 = smem_addr(&bars[NS]);
    const uint32_t emptyK0 = smem_addr(&bars[2 * NS]);
    const uint32_t emptyV0 = smem_addr(&bars[3 * NS]);
    const uint32_t sfull0 = smem_addr(&bars[4 * NS]);
    const uint32_t sfree0 = smem_addr(&bars[4 * NS + 2]);
    const uint32_t pfull0 = smem_addr(&bars[4 * NS + 4]);
    const uint32_t pvdone0 = smem_addr(&bars[4 * NS + 4 + C::NPB]);
    const uint32_t qready = smem_addr(&bars[4 * NS + 4 + 2 * C::NPB]);
    const uint32_t mmadone = smem_addr(&bars[4 * NS + 5 + 2 * C::NPB]);
    const uint32_t esync = smem_addr(&bars[4 * NS + 6 + 2 * C::NPB]);  // the softmax warps' own barrier

    if (warp == C::PRODUCER && lane == 0) {  // descriptors are parameters: fetch them before the wait
        tma_prefetch_desc(&tmKw);
        tma_prefetch_desc(&tmVw);
        if (a.has_deep) {
            tma_prefetch_desc(&tmKd);
            tma_prefetch_desc(&tmVd);
        }
    }
    if (tid == 0) {
        sflag[1] = 0;  // abort flag
        sflag[3] = 0;  // pairs this CTA merges at the end: sflag[4..5]
        for (int s = 0; s < NS; ++s) {
            mbar_init(fullK0 + 8 * s, 1);        // the producer's expect_tx
            mbar_init(fullV0 + 8 * s, 1);
            mbar_init(emptyK0 + 8 * s, 1 + nsw);  // the S commit and one arrival per softmax warp
            mbar_init(emptyV0 + 8 * s, 1);        // the P V commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull0 + 8 * b, 1);
            mbar_init(sfree0 + 8 * b, nst);
        }
        for (int b = 0; b < C::NPB; ++b) {
            mbar_init(pfull0 + 8 * b, nst);
            mbar_init(pvdone0 + 8 * b, 1);
        }
        mbar_init(qready, nst);
        mbar_init(mmadone, 1);
        mbar_init(esync, nst);
        mbar_fence_init();
    }
    // rows past a short box are never written by TMA; Q and P rows past the query count are never
    // written by the softmax: keep all of them finite (zero)
    {
        const bool short_box = pa.deep_box < kTileRows || pa.ring_box < kTileRows;
        uint4 *z = reinterpret_cast<uint4 *>(short_box ? stages : qs);
        const int n16 = (short_box ? NS * C::STAGE_BYTES : 0) / 16 + (C::Q_BYTES + C::NPB * C::P_BYTES) / 16;
        for (int i = tid; i < n16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
        fence_async_smem();
    }
    if (!a.early) pdl_wait();
    const ChunkPlan cp = plan_chunks(a, cum, Ts, sflag, tid, warp, lane);
    const int chunk = cp.chunk, pieces = cp.pieces, head = cp.head;
    const int g_begin = cp.g_begin, g_end = cp.g_end;
    if (g_begin >= g_end) {
        if (a.early) pdl_wait();  // the launch completes only after its predecessor
        return;
    }
    const int ntiles = g_end - g_begin;
    const int P_first = pieces ? head : pair_of(cum, N, kvH, g_begin);
    const uint32_t stage0 = smem_addr(stages);
    const uint32_t q0 = smem_addr(qs);
    const uint32_t p0 = smem_addr(ps);

    // ---- tensor memory: one warp allocates, every thread learns the base after the barrier
    if (warp == C::MMA_WARP) {
        tmem_alloc(smem_addr(&sflag[8]), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = static_cast<uint32_t>(sflag[8]);

    if (warp == C::PRODUCER) {
        // ================================================================ producer (one thread)
        if (lane == 0) {
            int n, kh, lt;
            SeqGeom sg;
            if (pieces) {
                n = N == 1 ? 0 : P_first / kvH;
                kh = P_first - n * kvH;
                sg = N == 1 ? cp.sg1 : seq_geom(Ts[n], pa);
                lt = (blockIdx.x - head * pieces) * chunk;
            } else {
                n = seq_of(cum, N, g_begin);
                sg = seq_geom(Ts[n], pa);
                const int rel = g_begin - cum[n];
                kh = rel / sg.total;
                lt = rel - kh * sg.total;
            }
            // K of tile t is loaded KA tiles ahead of V of tile t: the scores and the softmax of a
            // tile run while its V is still in flight, and neither half of a stage is held longer
            // than its consumer needs it.
            constexpr int KA = C::KA;
            int nk = 0, nv = 0;
            bool ok = true;
            bool waited = !a.early;
            while (nv < ntiles) {
                if (nk < ntiles && nk <= nv + KA) {
                    const int s = nk % NS;
                    if (nk >= NS && !mbar_wait_bounded(emptyK0 + 8 * s, ((nk / NS) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    if (*reinterpret_cast<volatile int *>(&sflag[1])) break;
                    const Tile t = tile_at(sg, lt, pa);
                    const bool deep = t.kind == kDeep;
                    if (!waited && !deep) {  // ring rows: the previous launch may be writing the block
                        pdl_wait();
                        waited = true;
                    }
                    const int rows = deep ? pa.deep_box : pa.ring_box;
                    const int z = deep ? ((a.layer * N + n) * kvH + kh)
                                       : (((a.layer * N + n) * a.R + t.plane) * kvH + kh);
                    if constexpr (kDebug) {
                        const bool bad =
                            t.cnt < 1 || t.cnt > rows ||
                            (deep ? (t.t0 < 0 || t.t0 + t.cnt > sg.D || sg.D > a.dbg_deep_rows ||
                                     z >= a.dbg_deep_pages)
                                  : (t.y < 0 || t.y + t.cnt > pa.ring_slots || t.t0 < sg.D ||
                                     t.t0 + t.cnt > (t.kind == kDual ? sg.T : sg.T + a.B) || z >= a.dbg_ring_pages ||
                                     (t.y - (t.t0 % pa.ring_slots) + pa.ring_slots) % pa.ring_slots != 0));
                        if (bad) atomicOr(a.err, RIPE_DEVERR_BOUNDS);
                    }
                    TileDesc &dsc = sdesc[s];
                    dsc.pair = n * kvH + kh; dsc.n = n; dsc.kh = kh; dsc.T = sg.T;
                    dsc.kind = t.kind; dsc.t0 = t.t0; dsc.cnt = t.cnt; dsc.plane = t.plane;
                    vsrc[s] = make_int2(t.y, z);
                    const uint32_t fb = fullK0 + 8 * s;
                    mbar_expect_tx(fb, C::NBOX * rows * 64);
                    const uint32_t kdst = stage0 + s * C::STAGE_BYTES;
#pragma unroll
                    for (int b = 0; b < C::NBOX; ++b)
                        tma_load_3d(kdst + b * kBoxBytes, deep ? &tmKd : &tmKw, fb, b * kBoxCols, t.y, z);
                    if (++lt == sg.total) {
                        lt = 0;
                        if (++kh == kvH) {
                            kh = 0;
                            if (++n < N) sg = seq_geom(Ts[n], pa);
                        }
                    }
                    ++nk;
                } else {
                    const int s = nv % NS;
                    if (nv >= NS && !mbar_wait_bounded(emptyV0 + 8 * s, ((nv / NS) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    if (*reinterpret_cast<volatile int *>(&sflag[1])) break;
                    // the K load of this tile wrote its descriptor; K of tile nv + NS, which rewrites it,
                    // is issued after this load
                    const bool deep = sdesc[s].kind == kDeep;
                    const int rows = deep ? pa.deep_box : pa.ring_box;
                    const int2 yz = vsrc[s];
                    const uint32_t fb = fullV0 + 8 * s;
                    mbar_expect_tx(fb, C::NBOX * rows * 64);
                    const uint32_t vdst = stage0 + s * C::STAGE_BYTES + C::NBOX * kBoxBytes;
#pragma unroll
                    for (int b = 0; b < C::NBOX; ++b)
                        tma_load_3d(vdst + b * kBoxBytes, deep ? &tmVd : &tmVw, fb, b * kBoxCols, yz.x, yz.y);
                    ++nv;
                }
            }
            if (!ok) {
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            }
            // drain: the last issue of every stage must land before the CTA exits
            for (int k = (nk > NS ? nk - NS : 0); k < nk; ++k) mbar_wait_bounded(fullK0 + 8 * (k % NS), (k / NS) & 1);
            for (int k = (nv > NS ? nv - NS : 0); k < nv; ++k) mbar_wait_bounded(fullV0 + 8 * (k % NS), (k / NS) & 1);
        }
    } else if (warp == C::MMA_WARP) {
        // ================================================================ MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_m64(64, false);  // S = Q K^T: B (K tile) K-major
            constexpr uint32_t idO = idesc_bf16_m64(D, true);    // O += P V: B (V tile) MN-major
            const uint32_t tS = tbase + C::S_COL, tO = tbase + C::O_COL;
            // Two event streams, served as they become ready: S of tile ns (its K half loaded, its S
            // buffer read out by the softmax warps, and for a new pair the queries in shared memory),
            // and P V of tile npv (its probabilities written and its V half loaded).  S thus runs up
            // to two tiles ahead of the softmax warps.
            int ns = 0, npv = 0, cur_pair = -1, npairs = 0;
            uint32_t first_bits = 0;  // bit t % 32: tile t opens its pair (ns - npv <= NS < 32)
            bool ok = true;
            unsigned long long t_idle = 0;
            int idle = 0;
            while (npv < ntiles) {
                bool progress = false;
                if (ns < ntiles) {
                    const int s = ns % NS, b = ns & 1;
                    if (mbar_test(fullK0 + 8 * s, (ns / NS) & 1) &&
                        (ns < 2 || mbar_test(sfree0 + 8 * b, ((ns >> 1) - 1) & 1))) {
                        const int pair = sdesc[s].pair;
                        const bool opens = pair != cur_pair;
                        if (!opens || mbar_test(qready, npairs & 1)) {
                            if (opens) {
                                ++npairs;
                                cur_pair = pair;
                                first_bits |= 1u << (ns & 31);
                            } else {
                                first_bits &= ~(1u << (ns & 31));
                            }
                            tc_fence_after();
                            const uint32_t kaddr = stage0 + s * C::STAGE_BYTES;
#pragma unroll
                            for (int ks = 0; ks < D / 16; ++ks) {
                                const uint32_t off = (ks >> 1) * kBoxBytes + (ks & 1) * 32;
                                tc_mma(tS + 64 * b, sw64_desc(q0 + off, 16, 512), sw64_desc(kaddr + off, 16, 512),
                                       idS, ks > 0 ? 1u : 0u);
                            }
                            tc_commit(sfull0 + 8 * b);
                            tc_commit(emptyK0 + 8 * s);
                            ++ns;
                            progress = true;
                        }
                    }
                }
                if (npv < ns && mbar_test(pfull0 + 8 * (npv % C::NPB), (npv / C::NPB) & 1) &&
                    mbar_test(fullV0 + 8 * (npv % NS), (npv / NS) & 1)) {
                    const int sj = npv % NS, bj = npv % C::NPB;
                    const bool first = (first_bits >> (npv & 31)) & 1u;
                    tc_fence_after();
                    const uint32_t vaddr = stage0 + sj * C::STAGE_BYTES + C::NBOX * kBoxBytes;
                    const uint32_t paddr = p0 + bj * C::P_BYTES;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {  // 16 keys per step
                        const uint64_t ad = sw64_desc(paddr + (kk >> 1) * kBoxBytes + (kk & 1) * 32, 16, 512);
                        const uint64_t bd = sw64_desc(vaddr + kk * 1024, kBoxBytes, 512);
                        tc_mma(tO, ad, bd, idO, (kk > 0 || !first) ? 1u : 0u);
                    }
                    tc_commit(pvdone0 + 8 * bj);
                    tc_commit(emptyV0 + 8 * sj);
                    ++npv;
                    progress = true;
                }
                if (progress) {
                    idle = 0;
                } else if (++idle == 64) {
                    t_idle = global_ns();
                } else if (idle > 64 && (idle & 63) == 0) {
                    if (global_ns() - t_idle > kWaitNs || *reinterpret_cast<volatile int *>(&sflag[1])) {
                        ok = false;
                        break;
                    }
                }
            }
            if (!ok) {
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            }
            // every MMA this thread issued has completed before tensor memory is freed
            tc_commit(mmadone);
            mbar_wait_bounded(mmadone, 0);
        }
    } else if (warp < nsw) {
        // ================================================================ softmax / epilogue
        // tcgen05.ld .16x256b on the M = 64 accumulator: thread t of warp w holds MMA rows
        // 16 w + t / 4 (h = 0) and 16 w + t / 4 + 8 (h = 1), at columns 8 k + 2 (t % 4) + {0, 1},
        // k = 0..7 of a 64-column tile: register 4 k + 2 h + e.  MMA row 16 w + l holds query row
        // w rpq + l (l < rpq; the others are padding).  Each row is spread over the four threads with
        // the same t / 4; its maximum and sums combine with two shuffles.
        const int rb = 16 * warp + (lane >> 2);  // MMA row of h = 0; h = 1 is rb + 8
        const int cq = 2 * (lane & 3);           // first column of the thread in each 8-column group
        bool live[2];
        int qi[2], jq[2], lq[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int r = (lane >> 2) + 8 * h;  // lane within the quadrant
            qi[h] = warp * rpq + r;             // the query row held there
            live[h] = r < rpq && qi[h] < a.Mq;
            jq[h] = live[h] ? a.j0 + qi[h] / a.g : a.j0;  // block position of the row
            lq[h] = live[h] ? pa.jloop[jq[h]] : -1;       // its loop
        }
        const uint32_t tq = tbase + (static_cast<uint32_t>(32 * warp) << 16);  // this warp's lane quadrant
        const bool ring_all_visible = pa.nloops == 1 && pa.dwin < 0;
        bool aborted = false;
        // a barrier of the softmax warps with a bounded wait (a thread that gave up elsewhere never
        // leaves the others waiting for good)
        uint32_t es_phase = 0;
        auto epi_sync = [&]() {
            mbar_arrive(esync);
            if (!mbar_wait_bounded(esync, es_phase & 1)) {
                aborted = true;
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            }
            ++es_phase;
        };
        auto give_up = [&]() {
            aborted = true;
            atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
        };
        auto part_slot_ok = [&](int p) {
            if (kDebug && static_cast<int>(blockIdx.x) + p >= a.dbg_part_slots) {
                atomicOr(a.err, RIPE_DEVERR_BOUNDS);
                return false;
            }
            return true;
        };
        // the CTAs holding tiles of pair p (returns how many)
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
        // The tile loop, for NH = 2 rows per thread (more than 32 query rows) or NH = 1 (the second
        // row of every thread is padding).
        auto tile_loop = [&](auto nh_c) {
            constexpr int NH = decltype(nh_c)::value;
            // per row: the reference maximum (base 2), and this thread's share of the sums of the fp32
            // probabilities (the log-sum-exp) and of the probabilities as rounded to bf16 for the P V
            // product (the output is a true weighted average of V with those weights)
            float m_ref[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f}, l_bf[2] = {0.f, 0.f};
            int cur_pair = -1, pair_start = 0;
            bool first = false;
            // write the finished pair: the output when this CTA saw all its keys, else a partial
            auto finalize = [&](int p, int last_tile, bool have) {
                const int n = p / kvH, kh = p - (p / kvH) * kvH;
                int c_first;
                const int nparts = parts_of(p, c_first);
                const bool sole = nparts == 1;
                if (have && !mbar_wait_bounded(pvdone0 + 8 * (last_tile % C::NPB), (last_tile / C::NPB) & 1)) give_up();
                const bool abort_now = aborted || *reinterpret_cast<volatile int *>(&sflag[1]) != 0;
                tc_fence_after();
                // the row sums over the four threads of the row
                float lb[2], lr[2];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    lb[h] = l_bf[h] + __shfl_xor_sync(0xffffffffu, l_bf[h], 1);
                    lb[h] += __shfl_xor_sync(0xffffffffu, lb[h], 2);
                    lr[h] = l_run[h] + __shfl_xor_sync(0xffffffffu, l_run[h], 1);
                    lr[h] += __shfl_xor_sync(0xffffffffu, lr[h], 2);
                }
                const int ROWS = part_rows(a.Mq);
                size_t orow[2], prow[2];
                float inv[2];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const int row = qi[h], jj = row / a.g;
                    orow[h] = (static_cast<size_t>(n) * a.qB + jj) * a.Hq + kh * a.g + (row - jj * a.g);
                    prow[h] = (static_cast<size_t>(blockIdx.x) + p) * ROWS + row;
                    inv[h] = lb[h] > 0.f ? 1.f / lb[h] : 0.f;
                }
                const bool write = !abort_now && have && (sole || part_slot_ok(p));
#pragma unroll 1
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t v[16];
                    tmem_ld_16x256b_x4(tq + C::O_COL + c0, v);  // every lane of the warp takes part
                    tmem_wait_ld();
                    if (!write) continue;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        if (!live[h]) continue;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int col = c0 + 8 * k + cq;
                            const float o0 = __uint_as_float(v[4 * k + 2 * h]), o1 = __uint_as_float(v[4 * k + 2 * h + 1]);
                            if (sole) {
                                const __nv_bfloat162 h2 = __floats2bfloat162_rn(o0 * inv[h], o1 * inv[h]);
                                *reinterpret_cast<__nv_bfloat162 *>(&a.out[orow[h] * D + col]) = h2;
                            } else {
                                *reinterpret_cast<float2 *>(&a.part_o[prow[h] * D + col]) = make_float2(o0, o1);
                            }
                        }
                    }
                }
                if (write && (lane & 3) == 0) {
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        if (!live[h]) continue;
                        if (sole) {
                            if (a.lse) a.lse[orow[h]] = (m_ref[h] + __log2f(lr[h])) * 0.69314718055994531f;
                        } else {
                            *reinterpret_cast<float4 *>(&a.part_ml[prow[h] * 4]) = make_float4(m_ref[h], lb[h], lr[h], 0.f);
                        }
                    }
                }
                epi_sync();  // every row's partial written
                if (!sole && !abort_now && tid == 0) {
                    __threadfence();
                    if (arrive_last(&a.counters[p], nparts, a.epoch)) {
                        __threadfence();
                        sflag[4 + sflag[3]] = p;  // merged at the end of this CTA's tiles
                        sflag[3] += 1;
                    }
                }
                tc_fence_before();
            };

            // one (sequence, kv head) tile: this thread's masks, scaled scores and row maxima
            auto scores = [&](const TileDesc &dsc, const uint32_t (&sv)[32], float (&x)[32], float (&mt)[2]) {
                const bool full_view =
                    dsc.cnt == kTileRows &&
                    (dsc.kind == kDeep ||
                     (dsc.kind == kRing && ring_all_visible && dsc.t0 + kTileRows - 1 <= dsc.T + a.j0 &&
                      (pa.mode_eff != 0 || dsc.t0 >= dsc.T + a.j0 + a.qB - 1 - pa.W)));
                int c_lo[2] = {0, 0}, c_hi[2];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    c_hi[h] = live[h] ? (full_view ? 63 : dsc.cnt - 1) : -1;
                    if (!full_view) {  // the keys a row sees form one range of columns
                        const int pq = dsc.T + jq[h];
                        if (dsc.kind == kRing) {
                            if (lq[h] != dsc.plane) c_hi[h] = -1;  // the ring at plane r serves only loop r's queries
                            c_hi[h] = min(c_hi[h], pq - dsc.t0);   // causal
                            if (pa.mode_eff == 0) c_lo[h] = max(0, min(dsc.T, pq - pa.W) - dsc.t0);  // block or window
                        } else if (dsc.kind == kDual) {
                            c_hi[h] = min(c_hi[h], pq - pa.W - 1 - dsc.t0);  // keys older than W for this query
                        }
                    }
                }
                float mx[2][4];
#pragma unroll
                for (int h = 0; h < NH; ++h)
#pragma unroll
                    for (int k = 0; k < 4; ++k) mx[h][k] = -INFINITY;
                if (full_view && live[0] && (NH == 1 || live[1])) {  // every key visible to both rows: no range checks
#pragma unroll
                    for (int k = 0; k < 8; ++k)
#pragma unroll
                        for (int h = 0; h < NH; ++h)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const float v = __uint_as_float(sv[4 * k + 2 * h + e]) * a.scale_log2;
                                x[4 * k + 2 * h + e] = v;
                                mx[h][k & 3] = fmaxf(mx[h][k & 3], v);
                            }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k)
#pragma unroll
                        for (int h = 0; h < NH; ++h)
#pragma unroll
                            for (int e = 0; e < 2; ++e) {
                                const int c = 8 * k + cq + e;
                                const float v = (c >= c_lo[h] && c <= c_hi[h])
                                                    ? __uint_as_float(sv[4 * k + 2 * h + e]) * a.scale_log2
                                                    : -INFINITY;
                                x[4 * k + 2 * h + e] = v;
                                mx[h][k & 3] = fmaxf(mx[h][k & 3], v);
                            }
                }
#pragma unroll
                for (int h = 0; h < NH; ++h) mt[h] = fmaxf(fmaxf(mx[h][0], mx[h][1]), fmaxf(mx[h][2], mx[h][3]));
            };
            // probabilities against the reference maximum: bf16 pairs pk[2 k + h] (row h, columns
            // 8 k + cq, + 1) and this thread's shares of both sums
            auto probs = [&](const float (&x)[32], uint32_t (&pk)[16]) {
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float mr = m_ref[h] == -INFINITY ? 0.f : m_ref[h];  // every x is -inf when m_ref is
                    float ls0 = 0.f, ls1 = 0.f, lb0 = 0.f, lb1 = 0.f;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const float p0 = exp2f(x[4 * k + 2 * h] - mr);
                        const float p1 = exp2f(x[4 * k + 2 * h + 1] - mr);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                        if (k & 1) { ls1 += p0 + p1; lb1 += __low2float(h2) + __high2float(h2); }
                        else { ls0 += p0 + p1; lb0 += __low2float(h2) + __high2float(h2); }
                        pk[2 * k + h] = *reinterpret_cast<const uint32_t *>(&h2);
                    }
                    l_run[h] += ls0 + ls1;
                    l_bf[h] += lb0 + lb1;
                }
            };
            // P (bf16, row-major, 64-byte swizzle, K-major) -> shared-memory buffer pb: 4 bytes per (row, group)
            auto write_p = [&](int pb, const uint32_t (&pk)[16]) {
                uint8_t *pbuf = ps + pb * C::P_BYTES;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const int row = rb + 8 * h;
                    uint8_t *prow_s = pbuf + row * 64 + 2 * cq;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int box = k >> 2, ch = (k & 3) ^ ((row >> 1) & 3);
                        *reinterpret_cast<uint32_t *>(prow_s + box * kBoxBytes + ch * 16) = pk[2 * k + h];
                    }
                }
            };

            // With RIPE_TC_PAIR, tiles are taken two at a time when both belong to the same (sequence,
            // kv head): their scores are processed interleaved (instruction-level parallelism for the
            // one warp per sub-partition) and one lazy-maximum update covers both.  Without it (the
            // default) one tile per iteration, which never waits for the next tile's K.
            int i = 0;
            while (i < ntiles) {
                const int s0 = i % NS;
                if (!mbar_wait_bounded(fullK0 + 8 * s0, (i / NS) & 1)) { give_up(); break; }
                const TileDesc dsc0 = sdesc[s0];
                // the descriptor is copied: the K half of this tile may be reloaded once S is computed
                __syncwarp();
                if (lane == 0) mbar_arrive(emptyK0 + 8 * s0);
                if (dsc0.pair != cur_pair) {
                    // (a CTA's tiles are consecutive in the concatenated lists: its pairs follow each
                    // other with no gap)
                    if (cur_pair >= 0) finalize(cur_pair, i - 1, true);
                    if (cur_pair < 0 && a.early) pdl_wait();  // the caller may be writing the queries
                    // this pair's queries -> shared memory (row-major, 64-byte swizzle, K-major): lane l < rpq
                    // of warp w writes query row w rpq + l into MMA row 16 w + l
                    cur_pair = dsc0.pair;
                    const int mrow = 16 * warp + lane, qrow = warp * rpq + lane;
                    if (lane < rpq && qrow < a.Mq) {
                        const int jj = qrow / a.g, hg = qrow - jj * a.g;
                        const uint4 *src = reinterpret_cast<const uint4 *>(
                            a.q + ((static_cast<size_t>(dsc0.n) * a.qB + jj) * a.Hq + dsc0.kh * a.g + hg) * D);
#pragma unroll
                        for (int c = 0; c < D / 8; ++c) {
                            const int box = c >> 2, ch = (c & 3) ^ ((mrow >> 1) & 3);
                            *reinterpret_cast<uint4 *>(qs + box * kBoxBytes + mrow * 64 + ch * 16) = __ldg(src + c);
                        }
                    }
                    fence_async_smem();
                    mbar_arrive(qready);
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        m_ref[h] = -INFINITY;
                        l_run[h] = 0.f;
                        l_bf[h] = 0.f;
                    }
                    first = true;
                    pair_start = i;
                }
                TileDesc dsc1 = dsc0;
                bool two = false;
                if (RIPE_TC_PAIR && i + 1 < ntiles) {
                    const int s1 = (i + 1) % NS;
                    if (!mbar_wait_bounded(fullK0 + 8 * s1, ((i + 1) / NS) & 1)) { give_up(); break; }
                    dsc1 = sdesc[s1];
                    two = dsc1.pair == dsc0.pair;
                    // (a tile left for the next iteration releases its K half then)
                    __syncwarp();
                    if (two && lane == 0) mbar_arrive(emptyK0 + 8 * s1);
                }
                // ---- S of the tile(s): 32 scores each
                uint32_t sv0[32], sv1[32];
                if (!mbar_wait_bounded(sfull0 + 8 * (i & 1), (i >> 1) & 1)) { give_up(); break; }
                tc_fence_after();
                tmem_ld_16x256b_x8(tq + C::S_COL + 64 * (i & 1), sv0);
                if (two) {
                    if (!mbar_wait_bounded(sfull0 + 8 * ((i + 1) & 1), ((i + 1) >> 1) & 1)) { give_up(); break; }
                    tc_fence_after();
                    tmem_ld_16x256b_x8(tq + C::S_COL + 64 * ((i + 1) & 1), sv1);
                }
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(sfree0 + 8 * (i & 1));
                if (two) mbar_arrive(sfree0 + 8 * ((i + 1) & 1));
                // ---- masks, maxima, the lazy reference (one update for both tiles)
                float x0[32], x1[32], mt0[2], mt1[2] = {-INFINITY, -INFINITY};
                scores(dsc0, sv0, x0, mt0);
                if (two) scores(dsc1, sv1, x1, mt1);
                // a row's reference moves only when its maximum exceeds it by more than kLazyMax,
                // which is so exactly when one of the row's four threads sees such a key: only then
                // are the maxima combined over those threads
                float alpha[2] = {1.f, 1.f}, mloc[2];
                bool over = false;
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    mloc[h] = fmaxf(mt0[h], mt1[h]);
                    over = over || mloc[h] > m_ref[h] + kLazyMax;  // also true for a finite maximum when m_ref is -inf
                }
                if (__any_sync(0xffffffffu, over)) {
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        float mt = mloc[h];
                        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
                        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
                        if (mt > m_ref[h] + kLazyMax) {
                            alpha[h] = m_ref[h] == -INFINITY ? 0.f : exp2f(m_ref[h] - mt);
                            m_ref[h] = mt;
                        }
                        l_run[h] *= alpha[h];
                        l_bf[h] *= alpha[h];
                    }
                }
                uint32_t pk0[16], pk1[16];
                probs(x0, pk0);
                if (two) probs(x1, pk1);
                // ---- P buffers i % 4 and (i + 1) % 4 were last read by the P V products of tiles i - 4
                // and i - 3: wait for the later one (a pair's first finalize waited for every earlier
                // product).  The product of tile i - 1 may still run: it is waited for only when O has to
                // be rescaled, which the lazy maximum makes rare.
                const bool rescale = !first && __any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f);
                if (i - 3 >= pair_start) {
                    if (!mbar_wait_bounded(pvdone0 + 8 * ((i - 3) % C::NPB), ((i - 3) / C::NPB) & 1)) { give_up(); break; }
                    tc_fence_after();
                }
                if (rescale) {
                    if (!mbar_wait_bounded(pvdone0 + 8 * ((i - 1) % C::NPB), ((i - 1) / C::NPB) & 1)) { give_up(); break; }
                    tc_fence_after();
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {  // this thread's part of its two rows of O
                        uint32_t v[16];
                        tmem_ld_16x256b_x4(tq + C::O_COL + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 4; ++k)
#pragma unroll
                            for (int h = 0; h < NH; ++h)
#pragma unroll
                                for (int e = 0; e < 2; ++e)
                                    v[4 * k + 2 * h + e] = __float_as_uint(__uint_as_float(v[4 * k + 2 * h + e]) * alpha[h]);
                        tmem_st_16x256b_x4(tq + C::O_COL + c0, v);
                    }
                    tmem_wait_st();
                }
                write_p(i % C::NPB, pk0);
                if (two) write_p((i + 1) % C::NPB, pk1);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(pfull0 + 8 * (i % C::NPB));
                if (two) mbar_arrive(pfull0 + 8 * ((i + 1) % C::NPB));
                first = false;
                i += two ? 2 : 1;
            }
            if (aborted) give_up();
            if (cur_pair >= 0) finalize(cur_pair, ntiles - 1, !aborted);
        };
        if (rpq > 8)
            tile_loop(std::integral_constant<int, 2>{});
        else
            tile_loop(std::integral_constant<int, 1>{});
        // ---- merge the partials of the pairs this CTA arrived at last (stage, Q and P buffers are free)
        epi_sync();
        if (*reinterpret_cast<volatile int *>(&sflag[1]) == 0) {
            const int nm = sflag[3];
            for (int k = 0; k < nm; ++k) {
                const int p = sflag[4 + k];
                const int n = p / kvH, kh = p - (p / kvH) * kvH;
                int c_first;
                const int nparts = parts_of(p, c_first);
                const int ROWS = part_rows(a.Mq);
                float *pw = reinterpret_cast<float *>(stages);  // [nparts][ROWS] m, then weights
                float *pl = pw + nparts * ROWS;                 // [nparts][ROWS] l
                for (int e = tid; e < nparts * a.Mq; e += nst) {
                    const int c = e / a.Mq, i = e - c * a.Mq;
                    const size_t prow = (static_cast<size_t>(c_first + c) + p) * ROWS + i;
                    const float2 ml = __ldcg(reinterpret_cast<const float2 *>(&a.part_ml[prow * 4]));
                    pw[c * ROWS + i] = ml.x;
                    pl[c * ROWS + i] = ml.y;
                }
                epi_sync();
                for (int i = tid; i < a.Mq; i += nst) {
                    float M = -INFINITY;
                    for (int c = 0; c < nparts; ++c) M = fmaxf(M, pw[c * ROWS + i]);
                    float L = 0.f, Ll = 0.f;
                    for (int c = 0; c < nparts; ++c) {
                        const float mk = pw[c * ROWS + i];
                        const float w = (mk == -INFINITY) ? 0.f : exp2f(mk - M);
                        pw[c * ROWS + i] = w;
                        L += w * pl[c * ROWS + i];
                        const size_t prow = (static_cast<size_t>(c_first + c) + p) * ROWS + i;
                        Ll += w * __ldcg(&a.part_ml[prow * 4 + 2]);
                    }
                    fin[i * 4] = M;
                    fin[i * 4 + 1] = L;
                    fin[i * 4 + 2] = Ll;
                }
                epi_sync();
                for (int e = tid; e < a.Mq * (D / 4); e += nst) {
                    const int i = e / (D / 4), c4x = e - i * (D / 4);
                    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
                    for (int c = 0; c < nparts; ++c) {
                        const float w = pw[c * ROWS + i];
                        const float4 v = __ldcg(reinterpret_cast<const float4 *>(
                            &a.part_o[((static_cast<size_t>(c_first + c) + p) * ROWS + i) * D + 4 * c4x]));
                        acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
                    }
                    const float invL = 1.f / fin[i * 4 + 1];
                    const int j = i / a.g, h = kh * a.g + (i - j * a.g);
                    const size_t orow = (static_cast<size_t>(n) * a.qB + j) * a.Hq + h;
                    __nv_bfloat162 *op = reinterpret_cast<__nv_bfloat162 *>(&a.out[orow * D + 4 * c4x]);
                    op[0] = __floats2bfloat162_rn(acc.x * invL, acc.y * invL);
                    op[1] = __floats2bfloat162_rn(acc.z * invL, acc.w * invL);
                    if (c4x == 0 && a.lse) a.lse[orow] = (fin[i * 4] + __log2f(fin[i * 4 + 2])) * 0.69314718055994531f;
                }
                if (tid == 0) a.counters[p] = 0;
                epi_sync();
            }
        }
    }
    // ---- every role is done with tensor memory: free it
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::MMA_WARP) tmem_dealloc(tbase, C::TMEM_COLS);
}

// ---------------------------------------------------------------- host side
template <int D>
struct TcInst {
    using C = TcCfg<D>;
    static constexpr auto kernel = ripe_verify_tc_kernel<D>;
    static constexpr int kMax = tc_smem_bytes(C::SMEM_FIXED, kMaxBatch);
    static_assert(kMax <= kSmemLimit, "the largest batch's shared memory must fit a CTA");
    static cudaError_t set_attr_max() {
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMax);
    }
    static cudaError_t launch(const LaunchTarget &t, int grid, const VerifyArgs &args, cudaStream_t s) {
        if (grid > C::MAX_PARTS) grid = C::MAX_PARTS;  // partial weights the end-of-CTA merge can hold
        VerifyArgs a = args;
        a.xpair = 0;
        return launch_pdl(kernel, dim3(grid), dim3(C::THREADS), tc_smem_bytes(C::SMEM_FIXED, t.N), s, *t.tmKd,
                          *t.tmVd, *t.tmKw, *t.tmVw, a);
    }
};

cudaError_t set_verify_tc_attributes() {
    cudaError_t e = TcInst<64>::set_attr_max();
    if (e == cudaSuccess) e = TcInst<96>::set_attr_max();
    if (e == cudaSuccess) e = TcInst<128>::set_attr_max();
    return e;
}

cudaError_t launch_verify_tc(int d, const LaunchTarget &t, int grid, const VerifyArgs &a, cudaStream_t s) {
    switch (d) {
        case 64: return TcInst<64>::launch(t, grid, a, s);
        case 96: return TcInst<96>::launch(t, grid, a, s);
        case 128: return TcInst<128>::launch(t, grid, a, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace ripe
