// Internal definitions shared by the verify kernels (sm_100a): the argument block, the tile
// descriptor a producer hands to its consumers, and how a launch cuts the tile lists of all
// (sequence, kv head) pairs into per-CTA chunks.
#pragma once

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
    int N, kvH, g, Hq, B, R, layer, Mq, min_chunk;
    // queries: block positions j0 .. j0 + qB - 1 (q, out, lse and the fused block hold qB rows
    // per sequence); a verification has j0 = 0, qB = B, a draft step j0 = its position, qB = 1
    int j0, qB;
    // launched as clusters of 2 CTAs: when each (sequence, kv head) is split into two pieces, the
    // CTA holding the second piece sends its partial to the first through distributed shared memory
    int xpair;
    int has_deep;  // the deepest-plane maps are valid (the full cache has no such region)
    // early start: the previous launch on the stream writes neither the lengths T nor the
    // deepest-plane region, so both are read, and deepest-plane tiles streamed, before waiting for
    // it (programmatic dependent launch); everything else waits
    int early;
    float scale_log2;
    // 0: the arrival counters start the launch at zero (the merging CTA clears each after use).
    // Otherwise the launch's epoch: a counter's top 16 bits tag the launch that last counted on it,
    // so counters left by an earlier launch count as zero and need no clearing in between.
    uint32_t epoch;
    // fused append (ripe_append_verify): block K/V [N][B][kvH][d] written to ring plane r
    const uint4 *blk_k, *blk_v;
    uint4 *ring_k, *ring_v;
    int max_T;
    // region sizes for the index checks of debug builds
    int dbg_deep_rows, dbg_part_slots;
    long long dbg_deep_pages, dbg_ring_pages;
};

constexpr int kSmemLimit = 232448;  // dynamic shared memory per CTA on sm_100
#ifndef RIPE_MAX_STAGES
#define RIPE_MAX_STAGES 8               // TMA pipeline depth cap (shared memory sets the rest)
#endif
#ifndef RIPE_MAX_STAGES_WIDE
// head_dim 128 with a single tile group (16-32-query rows per kv head, GQA): 3 stages of 32 KB
// measured faster than 2 or 4 on B200 (long-context GQA verify: 204 vs 230 / 218 us)
#define RIPE_MAX_STAGES_WIDE 3
#endif
#ifndef RIPE_MIN_CHUNK
#define RIPE_MIN_CHUNK 4                // at least this many 64-key tiles per CTA
#endif
constexpr float kLazyMax = 8.f;     // log2 headroom before the softmax reference moves
constexpr int kSwitchTiles = 3;     // tiles a CTA may add to its chunk to avoid a mid-stream head switch

struct TileDesc {
    int pair, n, kh, T, kind, t0, cnt, plane;
};

// One CTA's partial of pair p is published: true for the last of the nparts arrivals (that CTA
// merges them).  With an epoch (VerifyArgs::epoch) the count lives in the low 16 bits beside the
// epoch's low 16 bits; a CAS loop that only ever retries after another CTA's arrival succeeded.
__device__ __forceinline__ bool arrive_last(int32_t *counter, int nparts, uint32_t epoch) {
    if (epoch == 0) return atomicAdd(counter, 1) == nparts - 1;
    const uint32_t tag = (epoch & 0xFFFFu) << 16;
    uint32_t old = *reinterpret_cast<volatile uint32_t *>(counter);
    for (;;) {
        const uint32_t cnt = (old & 0xFFFF0000u) == tag ? (old & 0xFFFFu) : 0u;
        const uint32_t got = atomicCAS(reinterpret_cast<unsigned int *>(counter), old, tag | (cnt + 1));
        if (got == old) return static_cast<int>(cnt + 1) == nparts;
        old = got;
    }
}

// index of the last sequence whose first tile is <= gt
__device__ __forceinline__ int seq_of(const int *cum, int N, int gt) {
    int lo = 0, hi = N - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cum[mid] <= gt) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ int pair_of(const int *cum, int N, int kvH, int gt) {
    const int n = seq_of(cum, N, gt);
    const int tot = (cum[n + 1] - cum[n]) / kvH;
    return n * kvH + (gt - cum[n]) / tot;
}

// How a launch of `grid` CTAs cuts `total` tiles (tot0 per (sequence, kv head) when `same`):
// contiguous chunks of `chunk` tiles (pieces = 0), or, when several CTAs share each head,
// `pieces` equal pieces of every head, CTA c taking piece c % pieces of head c / pieces.
// Cuts fall on head boundaries when that costs at most kSwitchTiles tiles per CTA: a CTA then
// never switches to another head mid-stream.
__device__ __forceinline__ void choose_chunk(int total, int tot0, bool same, int grid, int N, int kvH, int min_chunk,
                                             int &chunk, int &pieces) {
    int ch = cdiv(total, grid);
    if (ch < min_chunk) ch = min_chunk;
    pieces = 0;
    if (same) {
        if (ch < tot0) {
            int P = grid / (N * kvH);
            if (P > tot0 / min_chunk) P = tot0 / min_chunk;
            if (P >= 1) {
                const int ca = cdiv(tot0, P);
                if (ca <= ch + kSwitchTiles) {
                    ch = ca;
                    pieces = P;
                }
            }
        } else {
            const int ca = cdiv(ch, tot0) * tot0;
            if (ca <= ch + kSwitchTiles) ch = ca;
        }
    }
    chunk = ch;
}

// Ring tile (index within the pair's list) holding position pos of the single-loop ring [D, T + B).
__device__ __forceinline__ int ring_tile_of(const SeqGeom &sg, const PlanArgs &pa, int pos) {
    const int o = pos - sg.D;
    return sg.nd + (o < sg.ring_first ? o / pa.ring_box : sg.nr1 + (o - sg.ring_first) / pa.ring_box);
}

// Where a verify launch reads from: the four tensor maps, the device and its SM count.
struct LaunchTarget {
    const CUtensorMap *tmKd, *tmVd, *tmKw, *tmVw;
    int device, num_sms, N;
};

// The tensor-core (tcgen05) consumer for 9..64 query rows per kv head (ripe_verify_tc.cu).
cudaError_t launch_verify_tc(int d, const LaunchTarget &t, int grid, const VerifyArgs &a, cudaStream_t s);
cudaError_t set_verify_tc_attributes();

// The chunk of the concatenated tile lists that this CTA streams.  Reads the lengths T (so the
// caller has waited for the kernel that writes them), fills Ts[N] and the per-sequence tile
// prefix sums cum[N + 1] in shared memory, and lets the next kernel in the stream be scheduled.
// Every thread of the CTA calls it (it synchronises the CTA).
struct ChunkPlan {
    int total, chunk, pieces;  // pieces 0: contiguous chunks of the whole tile list
    int tot_head;              // tiles per (sequence, kv head) in piece mode
    int head, g_begin, g_end;  // this CTA's head (piece mode) and tiles [g_begin, g_end)
    SeqGeom sg1;               // the sequence's geometry when N == 1
};

__device__ __forceinline__ ChunkPlan plan_chunks(const VerifyArgs &a, int *cum, int *Ts, int *sflag, int tid,
                                                 int warp, int lane) {
    const PlanArgs &pa = a.plan;
    const int N = a.N, kvH = a.kvH;
    ChunkPlan cp;
    cp.tot_head = 0;
    cp.sg1 = SeqGeom{};
    if (N == 1) {
        // one sequence: every thread reads T and cuts the list itself (no scan, no broadcast)
        const int T = a.T[0];
        cp.sg1 = seq_geom(T, pa);
        const int tot0 = cp.sg1.total;
        cp.tot_head = tot0;
        cp.total = tot0 * kvH;
        choose_chunk(cp.total, tot0, true, static_cast<int>(gridDim.x), 1, kvH, a.min_chunk, cp.chunk, cp.pieces);
        if (tid == 0) {
            Ts[0] = T;
            cum[0] = 0;
            cum[1] = cp.total;
        }
        __syncthreads();
        pdl_trigger();  // the next kernel may be scheduled; it waits for this one to finish
    } else {
        for (int n = tid; n < N; n += blockDim.x) {
            const int T = a.T[n];
            Ts[n] = T;
            cum[n + 1] = seq_geom(T, pa).total * kvH;
        }
        if (tid == 0) cum[0] = 0;
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
        pdl_trigger();
        cp.total = cum[N];
        if (warp == 0) {
            // equal tile counts for every (sequence, kv head)?
            bool same = true;
            for (int b = 0; b < N; b += 32) {
                const bool ok = (b + lane >= N) || (cum[b + lane + 1] - cum[b + lane] == cum[1]);
                same = same && __all_sync(0xffffffffu, ok);
            }
            if (lane == 0) {
                int ch, pc;
                choose_chunk(cp.total, cum[1] / kvH, same, static_cast<int>(gridDim.x), N, kvH, a.min_chunk, ch, pc);
                sflag[6] = ch;
                sflag[7] = pc;
            }
        }
        __syncthreads();
        cp.chunk = sflag[6];
        cp.pieces = sflag[7];
        if (cp.pieces) cp.tot_head = cum[1] / kvH;
    }
    cp.head = 0;
    if (cp.pieces) {
        cp.head = blockIdx.x / cp.pieces;
        cp.g_begin = cp.head * cp.tot_head + (blockIdx.x - cp.head * cp.pieces) * cp.chunk;
        cp.g_end = min(min(cp.g_begin + cp.chunk, (cp.head + 1) * cp.tot_head), cp.total);
    } else {
        cp.g_begin = blockIdx.x * cp.chunk;
        cp.g_end = min(cp.total, cp.g_begin + cp.chunk);
    }
    return cp;
}

}  // namespace ripe
