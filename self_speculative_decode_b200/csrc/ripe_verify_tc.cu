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
//   warps 0-3  softmax / epilogue.  Thread l < 16 of warp w owns query row i = 16 w + l: with the
//              MMA's M = 64 those rows sit in tensor-memory lanes 32 w + l.  Only ceil(rows / 16)
//              warps work.
//   warp 4     producer: one thread streams 64-key K/V tiles with 3-D TMA loads (no multicast)
//              into an NS-stage ring guarded by mbarriers, as in the mma.sync kernel.
//   warp 5     MMA: allocates tensor memory; one thread issues, per tile i,
//                S[i & 1] = Q K_i^T   (M = 64 query rows, N = 64 keys, K = head_dim)
//              and, once the softmax has written P_i (bf16, shared memory),
//                O += P_i V_i         (M = 64, N = head_dim, K = 64 keys; V read in place from the
//                                      TMA stage as an MN-major operand)
//              and frees the stage with tcgen05.commit.  S of tile i + 1 is issued before O of
//              tile i, so the tensor core works on the next tile while the softmax runs.
// The softmax keeps the row's running maximum m and sum l in registers (base 2).  The maximum
// moves only when a tile's maximum exceeds it by more than 8 (exact; the rescale of O, a
// tensor-memory read-modify-write of the thread's row, is then rare).  Rows past the query
// count are zero in Q and never written out.
#include <mutex>

#include "ripe_verify.cuh"

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
// 32 consecutive 32-bit columns of the warp's 32 tensor-memory lanes: thread l gets lane l
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
        "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]),
        "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),
        "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
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
    static constexpr int FIXED = MISC + Q_BYTES + 2 * P_BYTES + FIN_BYTES;
    static constexpr int AVAIL = kSmemLimit - FIXED - 4 * (2 * kMaxBatch + 2);
    static constexpr int NS = AVAIL / STAGE_BYTES > 8 ? 8 : AVAIL / STAGE_BYTES;
    static_assert(NS >= 3, "not enough shared memory for the pipeline");
    static constexpr int SMEM_FIXED = FIXED + NS * STAGE_BYTES;
    static_assert(SMEM_FIXED + 4 * (2 * kMaxBatch + 2) <= kSmemLimit, "shared memory");
    // the end-of-CTA merge keeps (m, l) of up to 256 partials x 64 rows in the stage buffers
    static_assert(NS * STAGE_BYTES >= 256 * MROWS * 2 * 4, "stage buffers too small for the merge");
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
    uint8_t *ps = qs + C::Q_BYTES;                               // P[2]
    float *fin = reinterpret_cast<float *>(ps + 2 * C::P_BYTES); // [64][4] merge M, L_out, L_lse
    uint64_t *bars = reinterpret_cast<uint64_t *>(fin + C::MROWS * 4);
    // full[NS] empty[NS] sfull[2] sfree[2] pfull[2] pvdone[2] qready mmadone esync
    TileDesc *sdesc = reinterpret_cast<TileDesc *>(bars + 2 * NS + 11);  // [NS]
    int *sflag = reinterpret_cast<int *>(sdesc + NS);                     // [16]; sflag[8] = TMEM base
    int *cum = sflag + 16;                                                // [N + 1]
    int *Ts = cum + a.N + 1;                                              // [N]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;
    const int nsw = (a.Mq + 15) >> 4;  // softmax warps with rows
    const int nst = nsw * 32;          // their threads

    const uint32_t full0 = smem_addr(&bars[0]);
    const uint32_t empty0 = smem_addr(&bars[NS]);
    const uint32_t sfull0 = smem_addr(&bars[2 * NS]);
    const uint32_t sfree0 = smem_addr(&bars[2 * NS + 2]);
    const uint32_t pfull0 = smem_addr(&bars[2 * NS + 4]);
    const uint32_t pvdone0 = smem_addr(&bars[2 * NS + 6]);
    const uint32_t qready = smem_addr(&bars[2 * NS + 8]);
    const uint32_t mmadone = smem_addr(&bars[2 * NS + 9]);
    const uint32_t esync = smem_addr(&bars[2 * NS + 10]);  // the softmax warps' own barrier

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
            mbar_init(smem_addr(&bars[s]), 1);       // full: the producer's expect_tx
            mbar_init(smem_addr(&bars[NS + s]), 1);  // empty: one tcgen05.commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(sfull0 + 8 * b, 1);
            mbar_init(sfree0 + 8 * b, nst);
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
        const int n16 = (short_box ? NS * C::STAGE_BYTES : 0) / 16 + (C::Q_BYTES + 2 * C::P_BYTES) / 16;
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
            int i = 0;
            bool ok = true;
            bool waited = !a.early;
            for (; i < ntiles; ++i) {
                const int s = i % NS;
                if (i >= NS && !mbar_wait_bounded(empty0 + 8 * s, ((i / NS) - 1) & 1)) {
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
                const CUtensorMap *mk = deep ? &tmKd : &tmKw;
                const CUtensorMap *mv = deep ? &tmVd : &tmVw;
                const int z = deep ? ((a.layer * N + n) * kvH + kh)
                                   : (((a.layer * N + n) * a.R + t.plane) * kvH + kh);
                if constexpr (kDebug) {
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
            }
            if (!ok) {
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            }
            // drain: the last issue of every stage must land before the CTA exits
            for (int k = (i > NS ? i - NS : 0); k < i; ++k) mbar_wait_bounded(full0 + 8 * (k % NS), (k / NS) & 1);
        }
    } else if (warp == C::MMA_WARP) {
        // ================================================================ MMA issue (one thread)
        if (lane == 0) {
            constexpr uint32_t idS = idesc_bf16_m64(64, false);  // S = Q K^T: B (K tile) K-major
            constexpr uint32_t idO = idesc_bf16_m64(D, true);    // O += P V: B (V tile) MN-major
            const uint32_t tS = tbase + C::S_COL, tO = tbase + C::O_COL;
            int cur_pair = -1, npairs = 0;
            int pending = -1;            // tile whose P V product is still to be issued
            bool pending_first = false;  // ... and whether it is the first tile of its pair
            bool ok = true;
            auto issue_pv = [&](int j, bool first) -> bool {
                const int sj = j % NS, bj = j & 1;
                if (!mbar_wait_bounded(pfull0 + 8 * bj, (j >> 1) & 1)) return false;
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
                tc_commit(empty0 + 8 * sj);
                return true;
            };
            for (int i = 0; i < ntiles && ok; ++i) {
                const int s = i % NS, b = i & 1;
                if (!mbar_wait_bounded(full0 + 8 * s, (i / NS) & 1)) { ok = false; break; }
                const int pair = sdesc[s].pair;
                bool first = false;
                if (pair != cur_pair) {
                    if (pending >= 0) {
                        if (!issue_pv(pending, pending_first)) { ok = false; break; }
                        pending = -1;
                    }
                    // the softmax warps have written this pair's queries into shared memory
                    if (!mbar_wait_bounded(qready, npairs & 1)) { ok = false; break; }
                    ++npairs;
                    cur_pair = pair;
                    first = true;
                }
                if (i >= 2 && !mbar_wait_bounded(sfree0 + 8 * b, ((i >> 1) - 1) & 1)) { ok = false; break; }
                tc_fence_after();
                const uint32_t kaddr = stage0 + s * C::STAGE_BYTES;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks >> 1) * kBoxBytes + (ks & 1) * 32;
                    tc_mma(tS + 64 * b, sw64_desc(q0 + off, 16, 512), sw64_desc(kaddr + off, 16, 512), idS,
                           ks > 0 ? 1u : 0u);
                }
                tc_commit(sfull0 + 8 * b);
                if (pending >= 0 && !issue_pv(pending, pending_first)) { ok = false; break; }
                pending = i;
                pending_first = first;
            }
            if (ok && pending >= 0) ok = issue_pv(pending, pending_first);
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
        const int row = 16 * warp + lane;              // query row of this thread (lane < 16)
        const bool live = lane < 16 && row < a.Mq;
        const int jq = live ? a.j0 + row / a.g : a.j0;  // block position of the row
        const int lq = live ? pa.jloop[jq] : -1;        // its loop
        const uint32_t trow = tbase + (static_cast<uint32_t>(32 * warp) << 16);
        const bool ring_all_visible = pa.nloops == 1 && pa.dwin < 0;
        // l_run sums the fp32 probabilities (the log-sum-exp); l_bf sums them as rounded to bf16 for
        // the P V product, so that the output is a true weighted average of V with those weights
        float m_ref = -INFINITY, l_run = 0.f, l_bf = 0.f;
        int cur_pair = -1, n_cur = 0, kh_cur = 0;
        bool first = false, aborted = false;
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
        // write the finished pair: the output when this CTA saw all its keys, else a partial
        auto finalize = [&](int p, int last_tile, bool have) {
            const int n = p / kvH, kh = p - (p / kvH) * kvH;
            int c_first;
            const int nparts = parts_of(p, c_first);
            const bool sole = nparts == 1;
            if (have && !mbar_wait_bounded(pvdone0 + 8 * (last_tile & 1), (last_tile >> 1) & 1)) {
                aborted = true;
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
            }
            const bool abort_now = aborted || *reinterpret_cast<volatile int *>(&sflag[1]) != 0;
            tc_fence_after();
            const int ROWS = part_rows(a.Mq);
            const int jj = row / a.g, h = kh * a.g + (row - jj * a.g);
            const size_t orow = (static_cast<size_t>(n) * a.qB + jj) * a.Hq + h;
            const size_t prow = (static_cast<size_t>(blockIdx.x) + p) * ROWS + row;
            const float inv = l_bf > 0.f ? 1.f / l_bf : 0.f;
#pragma unroll 1
            for (int c0 = 0; c0 < D; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(trow + C::O_COL + c0, v);  // every lane of the warp takes part
                tmem_wait_ld();
                if (!live || abort_now || !have) continue;
                if (sole) {
                    uint4 *op = reinterpret_cast<uint4 *>(&a.out[orow * D + c0]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]) * inv,
                                                                            __uint_as_float(v[8 * q + 2 * e + 1]) * inv);
                            w[e] = *reinterpret_cast<const uint32_t *>(&h2);
                        }
                        op[q] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                } else if (part_slot_ok(p)) {
                    float4 *pp = reinterpret_cast<float4 *>(&a.part_o[prow * D + c0]);
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        pp[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                            __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                }
            }
            if (live && !abort_now) {
                if (sole) {
                    if (a.lse) a.lse[orow] = have ? (m_ref + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
                } else if (part_slot_ok(p)) {
                    *reinterpret_cast<float4 *>(&a.part_ml[prow * 4]) =
                        have ? make_float4(m_ref, l_bf, l_run, 0.f) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
                }
            }
            epi_sync();  // every row's partial written
            if (!sole && !abort_now && tid == 0) {
                __threadfence();
                const int old = atomicAdd(&a.counters[p], 1);
                if (old == nparts - 1) {
                    __threadfence();
                    sflag[4 + sflag[3]] = p;  // merged at the end of this CTA's tiles
                    sflag[3] += 1;
                }
            }
            tc_fence_before();
        };

        for (int i = 0; i < ntiles; ++i) {
            const int s = i % NS, b = i & 1;
            if (!mbar_wait_bounded(full0 + 8 * s, (i / NS) & 1)) { aborted = true; break; }
            const TileDesc dsc = sdesc[s];
            if (dsc.pair != cur_pair) {
                // (a CTA's tiles are consecutive in the concatenated lists: its pairs follow each
                // other with no gap)
                if (cur_pair >= 0) finalize(cur_pair, i - 1, true);
                if (cur_pair < 0 && a.early) pdl_wait();  // the caller may be writing the queries
                // this pair's queries -> shared memory (row-major, 64-byte swizzle, K-major)
                cur_pair = dsc.pair;
                n_cur = dsc.n;
                kh_cur = dsc.kh;
                if (live) {
                    const int hg = row - (row / a.g) * a.g;
                    const uint4 *src = reinterpret_cast<const uint4 *>(
                        a.q + ((static_cast<size_t>(n_cur) * a.qB + (jq - a.j0)) * a.Hq + kh_cur * a.g + hg) * D);
#pragma unroll
                    for (int c = 0; c < D / 8; ++c) {
                        const int box = c >> 2, ch = (c & 3) ^ ((row >> 1) & 3);
                        *reinterpret_cast<uint4 *>(qs + box * kBoxBytes + row * 64 + ch * 16) = __ldg(src + c);
                    }
                }
                fence_async_smem();
                mbar_arrive(qready);
                m_ref = -INFINITY;
                l_run = 0.f;
                l_bf = 0.f;
                first = true;
            }
            // ---- S of this tile
            if (!mbar_wait_bounded(sfull0 + 8 * b, (i >> 1) & 1)) { aborted = true; break; }
            tc_fence_after();
            uint32_t sv[64];
            {
                uint32_t lo[32], hi[32];
                tmem_ld32(trow + C::S_COL + 64 * b, lo);
                tmem_ld32(trow + C::S_COL + 64 * b + 32, hi);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    sv[c] = lo[c];
                    sv[32 + c] = hi[c];
                }
            }
            tc_fence_before();
            mbar_arrive(sfree0 + 8 * b);
            // ---- masks, the tile maximum, the lazy reference
            const bool full_view =
                dsc.cnt == kTileRows &&
                (dsc.kind == kDeep ||
                 (dsc.kind == kRing && ring_all_visible && dsc.t0 + kTileRows - 1 <= dsc.T + a.j0 &&
                  (pa.mode_eff != 0 || dsc.t0 >= dsc.T + a.j0 + a.qB - 1 - pa.W)));
            const int pq = dsc.T + jq;
            float x[64];
            float mt = -INFINITY;
#pragma unroll
            for (int c = 0; c < 64; ++c) {
                float v = live ? __uint_as_float(sv[c]) * a.scale_log2 : -INFINITY;  // other lanes: unused
                if (!full_view) {
                    const int tpos = dsc.t0 + c;
                    bool vis = live && c < dsc.cnt;
                    if (dsc.kind == kRing)
                        vis = vis && lq == dsc.plane && tpos <= pq &&
                              (pa.mode_eff != 0 || tpos >= dsc.T || tpos >= pq - pa.W);
                    else if (dsc.kind == kDual)
                        vis = vis && tpos < pq - pa.W;
                    v = vis ? v : -INFINITY;
                }
                x[c] = v;
                mt = fmaxf(mt, v);
            }
            float alpha = 1.f;
            if (mt > m_ref + kLazyMax) {  // also true when m_ref is -inf and mt is finite
                alpha = m_ref == -INFINITY ? 0.f : exp2f(m_ref - mt);
                m_ref = mt;
            }
            l_run *= alpha;
            l_bf *= alpha;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) {
                const float p0 = m_ref == -INFINITY ? 0.f : exp2f(x[2 * c] - m_ref);
                const float p1 = m_ref == -INFINITY ? 0.f : exp2f(x[2 * c + 1] - m_ref);
                l_run += p0 + p1;
                const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
                l_bf += __low2float(h2) + __high2float(h2);
                pk[c] = *reinterpret_cast<const uint32_t *>(&h2);
            }
            // ---- the previous tile's P V product is done: P[b] is free and O is stable
            if (!first) {
                if (!mbar_wait_bounded(pvdone0 + 8 * ((i - 1) & 1), ((i - 1) >> 1) & 1)) { aborted = true; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, alpha != 1.f)) {  // rescale this thread's row of O
#pragma unroll 1
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t v[32];
                        tmem_ld32(trow + C::O_COL + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
                        tmem_st32(trow + C::O_COL + c0, v);
                    }
                    tmem_wait_st();
                }
            }
            // ---- P (bf16, row-major, 64-byte swizzle, K-major) -> shared memory
            if (lane < 16) {
                uint8_t *prow_s = ps + b * C::P_BYTES + row * 64;
#pragma unroll
                for (int k = 0; k < 8; ++k) {  // 8 keys per 16-byte chunk
                    const int box = k >> 2, ch = (k & 3) ^ ((row >> 1) & 3);
                    *reinterpret_cast<uint4 *>(prow_s + box * kBoxBytes + ch * 16) =
                        make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
                }
            }
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(pfull0 + 8 * b);
            first = false;
        }
        if (aborted) {
            atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
        }
        if (cur_pair >= 0) finalize(cur_pair, ntiles - 1, !aborted);
        // ---- merge the partials of the pairs this CTA arrived at last (stage buffers are free)
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
        if (grid > 256) grid = 256;  // the end-of-CTA merge keeps <= 256 partial weights per row
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
