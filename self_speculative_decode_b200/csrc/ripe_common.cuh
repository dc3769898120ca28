// Internal definitions shared by the RIPE library's translation units (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <vector>

#ifndef RIPE_NO_NVTX
#include <nvtx3/nvToolsExt.h>
#endif

#include "ripe.h"

namespace ripe {

// A named range around each C-ABI call for profilers (NVTX, header-only; a branch on a null
// function pointer when no tool is attached).  -DRIPE_NO_NVTX compiles it out.
struct NvtxRange {
#ifndef RIPE_NO_NVTX
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
#else
    explicit NvtxRange(const char *) {}
#endif
    NvtxRange(const NvtxRange &) = delete;
    NvtxRange &operator=(const NvtxRange &) = delete;
};

constexpr int kMaxBatch = 1024;   // sequences per cache (accepted lengths travel as kernel parameters)
constexpr int kMaxLoops = 256;    // R
constexpr int kTileRows = 64;     // keys per pipeline stage
constexpr int kBoxCols = 32;      // bf16 per TMA box row: 64 bytes, 64-byte swizzle
constexpr int kBoxBytes = kTileRows * 64;  // one box slot in shared memory (4 KB)
constexpr int kStages = 4;        // TMA pipeline depth of the verify kernel
constexpr int kMaxQueryRows = 64; // B * (Hq / kvH) per key/value head
constexpr int kMaxDevices = 64;   // devices a process may drive (per-device set-up tables)
// debug builds: bf16 bits written into key/value rows that hold no live position (the largest
// finite value: a masked read multiplies it by 0, any weighted read overflows the output)
constexpr int kPoisonByte = 0x7F;
#ifdef RIPE_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif

// Bounded waits: a kernel that does not see its copies land within this time records
// RIPE_DEVERR_WAIT_TIMEOUT and stops (it never traps).
constexpr unsigned long long kWaitNs = 4000000000ull;

struct HostIntArray {
    int32_t v[kMaxBatch];
};

}  // namespace ripe

// The opaque handle of the C ABI.
struct ripe_cache {
    // geometry
    int N, L, Hq, kvH, g, d, R, W, max_T, max_B, mode;
    int ring_slots;  // S = min(W + max_B, max_T)
    int deep_rows;   // max(0, max_T - W)
    int deep_box, ring_box;  // TMA box heights (<= 64)
    int device, num_sms;
    // device memory
    __nv_bfloat16 *Kd, *Vd;  // [L][N][kvH][deep_rows][d]
    __nv_bfloat16 *Kw, *Vw;  // [L][N][R][kvH][S][d]
    int32_t *T_dev;          // [N]
    uint32_t *err_dev;       // device error word
    float *part_o;           // [part_slots][part_rows][d]
    float *part_ml;          // [part_slots][part_rows][4]: m, l_out, l_lse, -
    int32_t *counters;       // [N * kvH] arrivals per (sequence, kv head), reset by the last arrival
    int part_slots, part_rows;
    CUtensorMap tm_Kd, tm_Vd, tm_Kw, tm_Vw;
    // host copy of the state
    std::vector<int32_t> T;   // committed lengths (an upper bound when !synced)
    int B_cur;                // block in flight (0 = none)
    std::vector<uint8_t> appended;  // [L][R] planes of the block appended
    std::vector<int> drafted;       // [L][R] draft positions written at each plane (before the block)
    bool prefix_set, synced;
    // the last launch on this cache wrote the lengths T or the deepest-plane region (commit with
    // eviction, prefix load): the next verify waits for it before reading either
    bool lengths_dirty;
    int64_t kv_bytes, scratch_bytes;
    int64_t launches;
};

namespace ripe {

// ---------------------------------------------------------------- tile plan
// The keys of one (sequence, kv head) at loop r form a list of tiles:
//   DEEP  the deepest-plane region, positions [0, D), D = max(0, T - W)
//   RING  positions [D, T + B) at plane r from the window ring (window + draft block), once
//         for every distinct loop r of the call (queries of other loops do not see it)
//   DUAL  positions [D, min(T, T + B - 1 - W)) at plane R-1 from the ring: window keys
//         that are older than W for the later queries of the block (query-relative rule)
// Ring ranges are cut where the ring wraps, so every tile is one box of consecutive slots.
enum TileKind { kDeep = 0, kRing = 1, kDual = 2 };

struct PlanArgs {
    int W, B, R, ring_slots, deep_box, ring_box, mode_eff;
    // windowed draft attention (dwin >= 0): the query of block position dj attends only to keys
    // t < sink and t >= T + dj - dwin; the deepest-plane tiles in between are not read
    int sink, dwin, dj;
    int nloops;                      // distinct loops of this call (1 for a single-loop verify)
    uint8_t loop[kMaxQueryRows];     // those loops; the ring is read once per loop
    uint8_t jloop[kMaxQueryRows];    // loop of each block position j
};

struct SeqGeom {
    int T, D, nd, s0;  // s0: ring slot of position D
    int se, nds, dw0;  // windowed draft: sink keys [0, se) in nds tiles, then deep keys [dw0, D)
    int ring_len, ring_first, nr1, nr;
    int dual_len, dual_first, ndl1, ndl;
    int total;
};

struct Tile {
    int kind, t0, cnt, y, plane;
};

__host__ __device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

// ceil(a / box) with the common box of 64 rows as a shift
__host__ __device__ __forceinline__ int ctiles(int a, int box) {
    return box == 64 ? (a + 63) >> 6 : cdiv(a, box);
}

__host__ __device__ __forceinline__ SeqGeom seq_geom(int T, const PlanArgs &a) {
    SeqGeom s;
    s.T = T;
    s.D = T - a.W > 0 ? T - a.W : 0;
    if (a.dwin >= 0) {
        s.se = a.sink < s.D ? a.sink : s.D;
        s.nds = ctiles(s.se, a.deep_box);
        const int ws = T + a.dj - a.dwin;
        s.dw0 = ws > s.se ? (ws < s.D ? ws : s.D) : s.se;
        s.nd = s.nds + ctiles(s.D - s.dw0, a.deep_box);
    } else {
        s.se = s.nds = s.dw0 = 0;
        s.nd = ctiles(s.D, a.deep_box);
    }
    s.s0 = s.D % a.ring_slots;
    s.ring_len = T + a.B - s.D;
    s.ring_first = s.ring_len < a.ring_slots - s.s0 ? s.ring_len : a.ring_slots - s.s0;
    s.nr1 = ctiles(s.ring_first, a.ring_box);
    s.nr = s.nr1 + ctiles(s.ring_len - s.ring_first, a.ring_box);
    int dl = 0;
    if (a.mode_eff == 0) {
        const int hi = T < T + a.B - 1 - a.W ? T : T + a.B - 1 - a.W;
        dl = hi - s.D > 0 ? hi - s.D : 0;
    }
    s.dual_len = dl;
    s.dual_first = dl < a.ring_slots - s.s0 ? dl : a.ring_slots - s.s0;
    s.ndl1 = ctiles(s.dual_first, a.ring_box);
    s.ndl = s.ndl1 + ctiles(s.dual_len - s.dual_first, a.ring_box);
    s.total = s.nd + a.nloops * s.nr + s.ndl;
    return s;
}

__host__ __device__ __forceinline__ Tile tile_at(const SeqGeom &s, int lt, const PlanArgs &a) {
    Tile t;
    if (lt < s.nd) {
        t.kind = kDeep;
        int end;
        if (lt < s.nds) {  // attention-sink tiles of a windowed draft
            t.t0 = lt * a.deep_box;
            end = s.se;
        } else {
            t.t0 = s.dw0 + (lt - s.nds) * a.deep_box;
            end = s.D;
        }
        t.cnt = (end - t.t0) < a.deep_box ? (end - t.t0) : a.deep_box;
        t.y = t.t0;
        t.plane = a.R - 1;
        return t;
    }
    lt -= s.nd;
    int len, first, n1;
    if (lt < a.nloops * s.nr) {
        int k = 0;
        while (lt >= s.nr) { lt -= s.nr; ++k; }
        len = s.ring_len; first = s.ring_first; n1 = s.nr1;
        t.kind = kRing; t.plane = a.loop[k];
    } else {
        lt -= a.nloops * s.nr;
        len = s.dual_len; first = s.dual_first; n1 = s.ndl1;
        t.kind = kDual; t.plane = a.R - 1;
    }
    int off, seg_end;
    if (lt < n1) {  // up to the end of the ring
        off = lt * a.ring_box;
        seg_end = first;
        t.y = s.s0 + off;
    } else {        // after the wrap, from slot 0
        off = first + (lt - n1) * a.ring_box;
        seg_end = len;
        t.y = off - first;
    }
    t.t0 = s.D + off;
    t.cnt = (seg_end - off) < a.ring_box ? (seg_end - off) : a.ring_box;
    return t;
}

// ---------------------------------------------------------------- PTX wrappers
#if defined(__CUDACC__)
__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for the phase with the given parity to complete; false after kWaitNs nanoseconds.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

// ---- register reallocation between warpgroups (all threads of a warpgroup execute the same one)
template <int N>
__device__ __forceinline__ void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---- thread-block clusters (a pair of CTAs exchanging partial results in shared memory)
// every thread of every CTA of the cluster: arrive (release) and wait (acquire)
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// shared::cluster address of the same shared-memory offset in CTA `rank` of this cluster
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_v2(uint32_t addr, float a, float b) {
    asm volatile("st.shared::cluster.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}

// asynchronous stores into another CTA's shared memory that count their bytes on its mbarrier
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(addr),
                 "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(addr),
                 "f"(a), "f"(b), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void fence_acq_rel_cluster() {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

// arrive on an mbarrier of another CTA of the cluster, releasing this thread's prior writes
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// bounded wait on a local mbarrier that another CTA of the cluster arrives on (acquire at cluster scope)
__device__ __forceinline__ bool mbar_wait_cluster_bounded(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = global_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i) {
            uint32_t ok;
            asm volatile(
                "{\n\t.reg .pred p;\n\t"
                "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
                "selp.u32 %0, 1, 0, p;\n\t}"
                : "=r"(ok)
                : "r"(bar), "r"(parity)
                : "memory");
            if (ok) return true;
        }
        if (global_ns() - t0 > kWaitNs) return false;
    }
}

// Bring a tensor-map descriptor (a kernel parameter) into the TMA unit's cache ahead of use.
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled TMA load (no multicast) completing on an mbarrier.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap *m, uint32_t bar, int x,
                                            int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                        uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                          uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr)
                 : "memory");
}

// D = A(16x16, bf16, row) * B(16x8, bf16, col) + D, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Transpose of an 8x8 bf16 matrix held one row-pair per lane (row lane/4, cols 2*(lane%4)+{0,1}).
__device__ __forceinline__ uint32_t movmatrix_t(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// Programmatic dependent launch: wait for the previous kernel in the stream to finish (and its
// memory to be visible) / allow the next kernel to be scheduled early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}
#endif

// Launch with programmatic stream serialization: the kernel may start while the previous one
// drains; every such kernel calls pdl_wait() before touching memory a previous kernel writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// The same with clusters of `cluster` CTAs along x (grid must be a multiple of it).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                               int cluster, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Most clusters of `cluster` CTAs of this kernel resident at once (0 if clusters cannot be used).
template <typename... KArgs>
int max_active_clusters(void (*kern)(KArgs...), dim3 block, size_t smem, int cluster, int grid_hint) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_hint);
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, reinterpret_cast<const void *>(kern), &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// ---------------------------------------------------------------- launchers (defined per .cu)
int launch_verify(ripe_cache *c, int layer, int r, const void *q, void *out, float *lse,
                  float scale, cudaStream_t s, const void *blk_k = nullptr, const void *blk_v = nullptr);
int launch_draft(ripe_cache *c, int layer, int r, int j, const void *k, const void *v, const void *q, void *out,
                 float *lse, float scale, cudaStream_t s, int sink = 0, int window = -1);
int launch_verify_wave(ripe_cache *c, int layer, const int32_t *loop_of_position, const void *q,
                       void *out, float *lse, float scale, cudaStream_t s);
int launch_append(ripe_cache *c, int layer, int r, int B, const void *k, const void *v,
                  cudaStream_t s);
int launch_commit(ripe_cache *c, const int32_t *acc_host, const int32_t *acc_dev, cudaStream_t s);
int launch_load_prefix(ripe_cache *c, int layer, int plane, const int32_t *T, const void *k,
                       const void *v, int64_t ld_t, cudaStream_t s);
int launch_export(ripe_cache *c, int n, int layer, void *k_out, void *v_out, uint8_t *present,
                  cudaStream_t s);
int launch_poison(ripe_cache *c, cudaStream_t s);  // debug builds: refill dead rows after a commit
// Raise the verify kernels' dynamic shared-memory limit on `device` (which must be current) to
// what the largest batch needs; once per device, thread-safe.
int ensure_verify_attributes(int device);
// ripe_set_verify_consumer: the consumer of verification launches with 9..64 query rows per kv head
int set_verify_consumer(int consumer);
int get_verify_consumer();

// Everything one verify launch needs, for callers that own the buffers and the scratch.
struct RawVerify {
    CUtensorMap tmKd, tmVd, tmKw, tmVw;
    const void *q;
    void *out;
    float *lse;
    const int32_t *T;
    float *part_o, *part_ml;
    int32_t *counters;
    uint32_t epoch;  // nonzero: epoch-tagged arrival counters (no clearing between launches)
    uint32_t *err;
    PlanArgs plan;
    int N, kvH, g, Hq, d, layer, grid, has_deep;
    int device, num_sms;
    int dbg_deep_rows;
    long long dbg_deep_pages, dbg_ring_pages;
    float scale;
};
int launch_verify_raw(const RawVerify &rv, cudaStream_t s);
int verify_rows_for(int Mq);  // query rows per partial slot for B * group query rows

}  // namespace ripe
