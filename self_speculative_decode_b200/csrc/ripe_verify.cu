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
//     ragged lengths and the three layouts (full, RIPE, deepest-only) balance the same way.
//   * One producer warp streams 64-key K/V tiles with 3-D TMA loads (64-byte swizzle, no
//     multicast) into a 4-stage shared-memory ring guarded by mbarriers.
//   * Consumer warps: each owns 16 query rows (B positions x GQA group, so one K/V read
//     serves the whole group) and 16 keys of each tile; S = Q K^T and O += P V run on the
//     tensor cores (mma.sync m16n8k16 bf16 -> fp32); fp32 online softmax in base 2 with
//     quad shuffles for the row max.
//   * A CTA that covers a whole (sequence, kv head) writes the output directly.  Otherwise
//     it writes an unnormalised partial (o, m, l); the last CTA to arrive (atomic counter,
//     no spinning) merges the partials by log-sum-exp and writes out / lse.
//   * Every wait is bounded: on timeout the kernel records RIPE_DEVERR_WAIT_TIMEOUT, drains
//     its own copies in flight and returns without writing results.
#include "ripe_common.cuh"

namespace ripe {

struct VerifyArgs {
    const __nv_bfloat16 *q;
    __nv_bfloat16 *out;
    float *lse;
    const int32_t *T;
    float *part_o;
    float *part_ml;
    int32_t *counters;
    uint32_t *err;
    PlanArgs plan;
    int N, kvH, g, Hq, B, R, layer, Mq, part_rows;
    float scale_log2;
};

template <int D, int WR>
struct VCfg {
    static constexpr int WK = (WR >= 4) ? 2 : 4;      // key groups per tile
    static constexpr int NCW = WR * WK;               // consumer warps
    static constexpr int THREADS = (NCW + 1) * 32;    // + one producer warp
    static constexpr int NBOX = D / kBoxCols;         // TMA boxes per K (or V) tile
    static constexpr int STAGE_BYTES = 2 * NBOX * kBoxBytes;
    static constexpr int MERGE_FLOATS = NCW * 16 * D;
    static constexpr int MLF = NCW * 16 * 2;
};

__host__ __device__ constexpr int verify_smem_fixed(int D, int WR) {
    return 1024 /* alignment slack */ + kStages * 2 * (D / kBoxCols) * kBoxBytes +
           ((WR >= 4 ? 2 : 4) * WR) * 16 * (D + 2) * 4 + 2 * kStages * 8 + 16 * 4;
}

int verify_smem_bytes(int d, int wr, int N) {
    return verify_smem_fixed(d, wr) + (2 * N + 2) * 4;
}

// Walks the concatenated tile lists in order.
struct TileIter {
    const int *cum;   // cum[n] = first global tile of sequence n
    const int *Ts;    // T per sequence
    int n, kh, lt;
    SeqGeom s;

    __device__ void start(int gt, int N, int kvH, const PlanArgs &a) {
        n = 0;
        while (n + 1 < N && cum[n + 1] <= gt) ++n;
        s = seq_geom(Ts[n], a);
        const int rel = gt - cum[n];
        kh = rel / s.total;
        lt = rel - kh * s.total;
    }
    __device__ void next(int N, int kvH, const PlanArgs &a) {
        if (++lt < s.total) return;
        lt = 0;
        if (++kh < kvH) return;
        kh = 0;
        if (++n < N) s = seq_geom(Ts[n], a);
    }
};

template <int D, int WR>
__global__ void __launch_bounds__(VCfg<D, WR>::THREADS, 1)
ripe_verify_kernel(const __grid_constant__ CUtensorMap tmKd, const __grid_constant__ CUtensorMap tmVd,
                   const __grid_constant__ CUtensorMap tmKw, const __grid_constant__ CUtensorMap tmVw,
                   const VerifyArgs a) {
    using C = VCfg<D, WR>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stages = base;
    float *mo = reinterpret_cast<float *>(base + kStages * C::STAGE_BYTES);  // [NCW][16][D]
    float *mml = mo + C::MERGE_FLOATS;                                       // [NCW][16][2]
    uint64_t *bars = reinterpret_cast<uint64_t *>(mml + C::MLF);             // full, empty
    int *sflag = reinterpret_cast<int *>(bars + 2 * kStages);                // [16]
    int *cum = sflag + 16;                                                   // [N + 1]
    int *Ts = cum + a.N + 1;                                                 // [N]

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;

    // ---- per-sequence tile counts and their prefix sums
    for (int n = tid; n < N; n += blockDim.x) {
        const int T = a.T[n];
        Ts[n] = T;
        cum[n + 1] = seq_geom(T, pa).total * kvH;
    }
    if (tid == 0) {
        cum[0] = 0;
        sflag[0] = 0;  // last-arrival flag
        sflag[1] = 0;  // abort flag
        for (int s = 0; s < kStages; ++s) {
            mbar_init(smem_addr(&bars[s]), 1);
            mbar_init(smem_addr(&bars[kStages + s]), C::NCW);
        }
        mbar_fence_init();
    }
    // rows past a short box are never written by TMA: keep them finite
    if (pa.deep_box < kTileRows || pa.ring_box < kTileRows) {
        uint4 *z = reinterpret_cast<uint4 *>(stages);
        for (int i = tid; i < kStages * C::STAGE_BYTES / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    }
    __syncthreads();
    if (warp == 0) {  // inclusive scan of cum[1..N] in chunks of 32
        int carry = 0;
        for (int b = 0; b < N; b += 32) {
            int v = (b + lane < N) ? cum[b + lane + 1] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, v, o);
                if (lane >= o) v += u;
            }
            if (b + lane < N) cum[b + lane + 1] = v + carry;
            carry += __shfl_sync(0xffffffffu, v, 31);
        }
    }
    __syncthreads();

    const int total = cum[N];
    const int chunk = cdiv(total, static_cast<int>(gridDim.x));
    const int g_begin = blockIdx.x * chunk;
    const int g_end = min(total, g_begin + chunk);
    if (g_begin >= g_end) return;

    const uint32_t full0 = smem_addr(&bars[0]);
    const uint32_t empty0 = smem_addr(&bars[kStages]);
    const uint32_t stage0 = smem_addr(stages);

    if (warp == C::NCW) {
        // ================================================================ producer
        if (lane == 0) {
            tma_prefetch_desc(&tmKd); tma_prefetch_desc(&tmVd);
            tma_prefetch_desc(&tmKw); tma_prefetch_desc(&tmVw);
            TileIter it;
            it.cum = cum; it.Ts = Ts;
            it.start(g_begin, N, kvH, pa);
            int i = 0;
            bool ok = true;
            for (int gt = g_begin; gt < g_end; ++gt, ++i) {
                const int s = i % kStages;
                if (i >= kStages && !mbar_wait_bounded(empty0 + 8 * s, ((i / kStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                const Tile t = tile_at(it.s, it.lt, pa);
                const bool deep = t.kind == kDeep;
                const int rows = deep ? pa.deep_box : pa.ring_box;
                const CUtensorMap *mk = deep ? &tmKd : &tmKw;
                const CUtensorMap *mv = deep ? &tmVd : &tmVw;
                const int z = deep ? ((a.layer * N + it.n) * kvH + it.kh)
                                   : (((a.layer * N + it.n) * a.R + t.plane) * kvH + it.kh);
                const uint32_t fb = full0 + 8 * s;
                mbar_expect_tx(fb, 2 * C::NBOX * rows * 64);
                const uint32_t kdst = stage0 + s * C::STAGE_BYTES;
                const uint32_t vdst = kdst + C::NBOX * kBoxBytes;
#pragma unroll
                for (int b = 0; b < C::NBOX; ++b) {
                    tma_load_3d(kdst + b * kBoxBytes, mk, fb, b * kBoxCols, t.y, z);
                    tma_load_3d(vdst + b * kBoxBytes, mv, fb, b * kBoxCols, t.y, z);
                }
                it.next(N, kvH, pa);
            }
            if (!ok) {
                atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
                // drain: the last issue of every stage must land before the CTA exits
                for (int k = (i > kStages ? i - kStages : 0); k < i; ++k)
                    mbar_wait_bounded(full0 + 8 * (k % kStages), (k / kStages) & 1);
            }
        }
        // the producer warp takes part in no consumer barrier (id 1)
        return;
    }

    // ==================================================================== consumers
    const int rg = warp / C::WK;   // row group: query rows 16*rg .. 16*rg + 15
    const int kg = warp % C::WK;   // key group: 16-key sub-blocks kg, kg + WK, ...
    const int g4 = lane >> 2, c4 = lane & 3;
    const int ctid = tid;          // consumers are threads 0 .. NCW*32 - 1
    const int nct = C::NCW * 32;

    // query rows held by this thread: i = 16*rg + g4 (+8); row i is block position i / g
    int jrow[2];
    bool rvalid[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = 16 * rg + g4 + 8 * h;
        rvalid[h] = i < a.Mq;
        jrow[h] = rvalid[h] ? i / a.g : a.B - 1;
    }
    // ldmatrix lane geometry (64-byte swizzle: 16-byte chunk ^= (row >> 1) & 3)
    const int mi = lane >> 3, r8 = lane & 7;
    const uint32_t swz = static_cast<uint32_t>(r8 >> 1);
    const int krow_off = (mi >> 1) * 8 + r8;  // K: matrices (keys 0-7 | 8-15) x (d lo | hi)
    const uint32_t kcol_sel = mi & 1;
    const int vrow_off = (mi & 1) * 8 + r8;   // V (trans): (keys 0-7 | 8-15) x (dv lo | hi)
    const uint32_t vcol_sel = mi >> 1;

    float o[D / 8][4];
    float m_run[2], l_run[2];
    uint32_t qa[D / 16][4];

    TileIter it;
    it.cum = cum; it.Ts = Ts;
    it.start(g_begin, N, kvH, pa);
    int cur_pair = -1, cur_n = 0, cur_kh = 0;
    bool aborted = false;

    auto load_q = [&](int n, int kh) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = 16 * rg + g4 + 8 * h;
            const uint32_t *qp = nullptr;
            if (rvalid[h]) {
                const int j = i / a.g, hg = i - (i / a.g) * a.g;
                qp = reinterpret_cast<const uint32_t *>(
                    a.q + ((static_cast<size_t>(n) * a.B + j) * a.Hq + kh * a.g + hg) * D);
            }
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
                qa[ks][h] = qp ? __ldg(qp + (16 * ks + 2 * c4) / 2) : 0u;
                qa[ks][2 + h] = qp ? __ldg(qp + (16 * ks + 8 + 2 * c4) / 2) : 0u;
            }
        }
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
    };

    auto finalize = [&](int n, int kh) {
        const int P = n * kvH + kh;
        // complete the row sums over the quad
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
        }
        float *mw = mo + warp * 16 * D;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
            *reinterpret_cast<float2 *>(&mw[g4 * D + 8 * nt + 2 * c4]) = make_float2(o[nt][0], o[nt][1]);
            *reinterpret_cast<float2 *>(&mw[(g4 + 8) * D + 8 * nt + 2 * c4]) = make_float2(o[nt][2], o[nt][3]);
        }
        if (c4 == 0) {
            mml[(warp * 16 + g4) * 2] = m_run[0];
            mml[(warp * 16 + g4) * 2 + 1] = l_run[0];
            mml[(warp * 16 + g4 + 8) * 2] = m_run[1];
            mml[(warp * 16 + g4 + 8) * 2 + 1] = l_run[1];
        }
        named_bar_sync(1, nct);
        const bool abort_now = *reinterpret_cast<volatile int *>(&sflag[1]) != 0;
        const int tot_n = (cum[n + 1] - cum[n]) / kvH;
        const int start = cum[n] + kh * tot_n;
        const int c_first = start / chunk, c_last = (start + tot_n - 1) / chunk;
        const int nparts = c_last - c_first + 1;
        const bool sole = nparts == 1;
        const int rows = WR * 16;
        for (int e = ctid; e < rows * D; e += nct) {
            const int i = e / D, col = e - (e / D) * D;
            const int rgi = i >> 4, row = i & 15;
            float M = -INFINITY;
#pragma unroll
            for (int k = 0; k < C::WK; ++k) M = fmaxf(M, mml[((rgi * C::WK + k) * 16 + row) * 2]);
            float acc = 0.f, L = 0.f;
            if (M != -INFINITY) {
#pragma unroll
                for (int k = 0; k < C::WK; ++k) {
                    const int w = rgi * C::WK + k;
                    const float mk = mml[(w * 16 + row) * 2];
                    if (mk != -INFINITY) {
                        const float f = exp2f(mk - M);
                        acc += mo[(w * 16 + row) * D + col] * f;
                        L += mml[(w * 16 + row) * 2 + 1] * f;
                    }
                }
            }
            if (abort_now) continue;
            if (sole) {
                if (i < a.Mq) {
                    const int j = i / a.g, h = kh * a.g + (i - j * a.g);
                    const size_t orow = (static_cast<size_t>(n) * a.B + j) * a.Hq + h;
                    a.out[orow * D + col] = __float2bfloat16_rn(acc / L);
                    if (col == 0 && a.lse) a.lse[orow] = (M + __log2f(L)) * 0.69314718055994531f;
                }
            } else {
                const size_t prow = (static_cast<size_t>(blockIdx.x) + P) * a.part_rows + i;
                a.part_o[prow * D + col] = acc;
                if (col == 0) {
                    a.part_ml[prow * 2] = M;
                    a.part_ml[prow * 2 + 1] = L;
                }
            }
        }
        if (!sole && !abort_now) {
            __threadfence();
            named_bar_sync(1, nct);
            if (ctid == 0) {
                const int old = atomicAdd(&a.counters[P], 1);
                sflag[0] = (old == nparts - 1) ? 1 : 0;
            }
            named_bar_sync(1, nct);
            if (sflag[0]) {
                __threadfence();
                for (int e = ctid; e < a.Mq * D; e += nct) {
                    const int i = e / D, col = e - (e / D) * D;
                    float M = -INFINITY;
                    for (int c = c_first; c <= c_last; ++c)
                        M = fmaxf(M, __ldcg(&a.part_ml[((static_cast<size_t>(c) + P) * a.part_rows + i) * 2]));
                    float acc = 0.f, L = 0.f;
                    for (int c = c_first; c <= c_last; ++c) {
                        const size_t prow = (static_cast<size_t>(c) + P) * a.part_rows + i;
                        const float mk = __ldcg(&a.part_ml[prow * 2]);
                        if (mk != -INFINITY) {
                            const float f = exp2f(mk - M);
                            acc += __ldcg(&a.part_o[prow * D + col]) * f;
                            L += __ldcg(&a.part_ml[prow * 2 + 1]) * f;
                        }
                    }
                    const int j = i / a.g, h = kh * a.g + (i - j * a.g);
                    const size_t orow = (static_cast<size_t>(n) * a.B + j) * a.Hq + h;
                    a.out[orow * D + col] = __float2bfloat16_rn(acc / L);
                    if (col == 0 && a.lse) a.lse[orow] = (M + __log2f(L)) * 0.69314718055994531f;
                }
                if (ctid == 0) a.counters[P] = 0;
            }
        }
        named_bar_sync(1, nct);  // the merge buffer is rewritten by the next pair
    };

    int i = 0;
    for (int gt = g_begin; gt < g_end; ++gt, ++i) {
        const int P = it.n * kvH + it.kh;
        if (P != cur_pair) {
            if (cur_pair >= 0) finalize(cur_n, cur_kh);
            cur_pair = P; cur_n = it.n; cur_kh = it.kh;
            load_q(cur_n, cur_kh);
        }
        const int s = i % kStages;
        if (!aborted && !mbar_wait_bounded(full0 + 8 * s, (i / kStages) & 1)) {
            aborted = true;
            atomicOr(a.err, RIPE_DEVERR_WAIT_TIMEOUT);
            *reinterpret_cast<volatile int *>(&sflag[1]) = 1;
        }
        if (!aborted) {
            const Tile t = tile_at(it.s, it.lt, pa);
            const int T = it.s.T;
            const uint32_t kbase = stage0 + s * C::STAGE_BYTES;
            const uint32_t vbase = kbase + C::NBOX * kBoxBytes;
#pragma unroll
            for (int kb0 = 0; kb0 < 4 / C::WK; ++kb0) {
                const int kb = kg + kb0 * C::WK;
                if (16 * kb >= t.cnt) break;
                // ---- S = Q K^T for 16 keys
                float S[2][4];
#pragma unroll
                for (int x = 0; x < 2; ++x) S[x][0] = S[x][1] = S[x][2] = S[x][3] = 0.f;
                const uint32_t krow = static_cast<uint32_t>(16 * kb + krow_off);
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t col16 = static_cast<uint32_t>(2 * (ks & 1)) + kcol_sel;
                    const uint32_t addr = kbase + (ks >> 1) * kBoxBytes + krow * 64 + ((col16 ^ swz) << 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(addr, b0, b1, b2, b3);
                    mma_16816(S[0], qa[ks], b0, b1);
                    mma_16816(S[1], qa[ks], b2, b3);
                }
                // ---- mask, scale, online softmax (base 2)
                float pr[2][4];
                float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int h = e >> 1;
                        const int kk = 16 * kb + 8 * nt + 2 * c4 + (e & 1);
                        const int tpos = t.t0 + kk;
                        const int p = T + jrow[h];
                        bool vis = kk < t.cnt;
                        if (t.kind == kRing)
                            vis = vis && tpos <= p && (pa.mode_eff != 0 || tpos >= T || tpos >= p - pa.W);
                        else if (t.kind == kDual)
                            vis = vis && tpos < p - pa.W;
                        const float x = vis ? S[nt][e] * a.scale_log2 : -INFINITY;
                        pr[nt][e] = x;
                        mt[h] = fmaxf(mt[h], x);
                    }
                float alpha[2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 1));
                    mt[h] = fmaxf(mt[h], __shfl_xor_sync(0xffffffffu, mt[h], 2));
                    const float mn = fmaxf(m_run[h], mt[h]);
                    alpha[h] = (mn == -INFINITY) ? 1.f : exp2f(m_run[h] - mn);
                    m_run[h] = mn;
                }
                uint32_t pa_frag[4];
                float lsum[2] = {0.f, 0.f};
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        const float mn = m_run[hh];
                        const float p0 = (mn == -INFINITY) ? 0.f : exp2f(pr[nt][2 * hh] - mn);
                        const float p1 = (mn == -INFINITY) ? 0.f : exp2f(pr[nt][2 * hh + 1] - mn);
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(p0, p1);
                        const float2 pf = __bfloat1622float2(pb);
                        lsum[hh] += pf.x + pf.y;
                        pa_frag[2 * nt + hh] = *reinterpret_cast<const uint32_t *>(&pb);
                    }
#pragma unroll
                for (int h = 0; h < 2; ++h) l_run[h] = l_run[h] * alpha[h] + lsum[h];
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt) {
                    o[nt][0] *= alpha[0]; o[nt][1] *= alpha[0];
                    o[nt][2] *= alpha[1]; o[nt][3] *= alpha[1];
                }
                // ---- O += P V for 16 keys
                const uint32_t vrow = static_cast<uint32_t>(16 * kb + vrow_off);
#pragma unroll
                for (int dv = 0; dv < D / 16; ++dv) {
                    const uint32_t col16 = static_cast<uint32_t>(2 * (dv & 1)) + vcol_sel;
                    const uint32_t addr = vbase + (dv >> 1) * kBoxBytes + vrow * 64 + ((col16 ^ swz) << 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(addr, b0, b1, b2, b3);
                    mma_16816(o[2 * dv], pa_frag, b0, b1);
                    mma_16816(o[2 * dv + 1], pa_frag, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty0 + 8 * s);
        }
        it.next(N, kvH, pa);
    }
    if (cur_pair >= 0) finalize(cur_n, cur_kh);
}

template <int D, int WR>
static cudaError_t set_attr_one(int N) {
    return cudaFuncSetAttribute(ripe_verify_kernel<D, WR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                verify_smem_bytes(D, WR, N));
}

int set_verify_attributes(int d, int N) {
    cudaError_t e = cudaSuccess;
    switch (d) {
        case 64: e = set_attr_one<64, 1>(N); if (!e) e = set_attr_one<64, 2>(N); if (!e) e = set_attr_one<64, 4>(N); break;
        case 96: e = set_attr_one<96, 1>(N); if (!e) e = set_attr_one<96, 2>(N); if (!e) e = set_attr_one<96, 4>(N); break;
        case 128: e = set_attr_one<128, 1>(N); if (!e) e = set_attr_one<128, 2>(N); if (!e) e = set_attr_one<128, 4>(N); break;
        default: return RIPE_EINVAL;
    }
    return e == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

template <int D, int WR>
static void launch_one(const ripe_cache *c, int grid, const VerifyArgs &a, cudaStream_t s) {
    ripe_verify_kernel<D, WR><<<grid, VCfg<D, WR>::THREADS, verify_smem_bytes(D, WR, c->N), s>>>(
        c->tm_Kd, c->tm_Vd, c->tm_Kw, c->tm_Vw, a);
}

int launch_verify(ripe_cache *c, int layer, int r, const void *q, void *out, float *lse, float scale,
                  cudaStream_t s) {
    VerifyArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.T = c->T_dev;
    a.part_o = c->part_o;
    a.part_ml = c->part_ml;
    a.counters = c->counters;
    a.err = c->err_dev;
    a.plan.W = c->W;
    a.plan.B = c->B_cur;
    a.plan.R = c->R;
    a.plan.r = r;
    a.plan.ring_slots = c->ring_slots;
    a.plan.deep_box = c->deep_box;
    a.plan.ring_box = c->ring_box;
    // at the deepest loop every key reads plane R-1, so the window rule changes nothing
    a.plan.mode_eff = (c->mode == RIPE_WINDOW_CACHE_RELATIVE || r == c->R - 1) ? 1 : 0;
    a.N = c->N;
    a.kvH = c->kvH;
    a.g = c->g;
    a.Hq = c->Hq;
    a.B = c->B_cur;
    a.R = c->R;
    a.layer = layer;
    a.Mq = c->B_cur * c->g;
    const int wr = a.Mq <= 16 ? 1 : (a.Mq <= 32 ? 2 : 4);
    a.part_rows = 16 * wr;
    a.scale_log2 = scale * 1.4426950408889634f;

    // grid: one CTA per SM, fewer when the host copy of T says there is less work
    int grid = c->num_sms;
    if (c->synced) {
        long total = 0;
        for (int n = 0; n < c->N; ++n) total += static_cast<long>(seq_geom(c->T[n], a.plan).total) * c->kvH;
        if (total < grid) grid = static_cast<int>(total);
    }
    if (grid < 1) grid = 1;
    switch (c->d * 8 + wr) {
        case 64 * 8 + 1: launch_one<64, 1>(c, grid, a, s); break;
        case 64 * 8 + 2: launch_one<64, 2>(c, grid, a, s); break;
        case 64 * 8 + 4: launch_one<64, 4>(c, grid, a, s); break;
        case 96 * 8 + 1: launch_one<96, 1>(c, grid, a, s); break;
        case 96 * 8 + 2: launch_one<96, 2>(c, grid, a, s); break;
        case 96 * 8 + 4: launch_one<96, 4>(c, grid, a, s); break;
        case 128 * 8 + 1: launch_one<128, 1>(c, grid, a, s); break;
        case 128 * 8 + 2: launch_one<128, 2>(c, grid, a, s); break;
        case 128 * 8 + 4: launch_one<128, 4>(c, grid, a, s); break;
        default: return RIPE_EINVAL;
    }
    c->launches += 1;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

}  // namespace ripe
