// Allocation-free verification attention: ripe_verify_attn_static (declared in include/ripe.h).
//
// For callers that cannot call cudaMalloc (their device memory belongs to an engine's pool or
// a framework, or they run while a stream capture is open).  The caller owns the cache buffers
// and the outputs; the kernel's scratch -- the partial (o, m, l) of each split key range and
// the per-(sequence, kv head) arrival counters -- lives in one file-scope device array of
// RIPE_STATIC_SCRATCH_BYTES that every GPU loading the library holds until the process exits.
// The kernel is the same one ripe_verify_attn launches.
#include <atomic>
#include <cstring>
#include <mutex>

#include "ripe_common.cuh"

namespace {

using ripe::kMaxDevices;

__device__ __align__(256) unsigned char g_static_scratch[RIPE_STATIC_SCRATCH_BYTES];

struct DeviceSetup {
    bool done;
    unsigned char *scratch;  // device address of g_static_scratch on this device
    int num_sms;
    std::atomic<uint32_t> epoch;  // of the last call on this device (tags the arrival counters)
};
DeviceSetup g_setup[kMaxDevices];
std::mutex g_setup_mu;

// Once per device, with that device current: the array's device address, the SM count, and the
// verify kernels' shared-memory limit.
// (In host code the array's name is only a host-side stand-in, never a device address.)
int setup_device(int dev, DeviceSetup *&out) {
    if (dev < 0 || dev >= kMaxDevices) return RIPE_EINVAL;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup &s = g_setup[dev];
    if (!s.done) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return RIPE_ECUDA;
        }
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
            cudaGetLastError();
            return RIPE_ECUDA;
        }
        // the kernels' shared-memory limit (shared with caches on this device; only ever raised)
        const int st = ripe::ensure_verify_attributes(dev);
        if (st != RIPE_OK) return st;
        s.scratch = static_cast<unsigned char *>(p);
        s.num_sms = sms;
        s.done = true;
    }
    out = &s;
    return RIPE_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The same 3-D bf16 map the cache uses: [pages][rows][d], box 32 elements x box_rows x 1, 64B swizzle.
bool encode(CUtensorMap *m, const void *base, int d, int rows, long long pages, int box_rows) {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(pages)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * 2 * rows};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(ripe::kBoxCols), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Encoded tensor maps of the views seen last (encoding four maps costs a few microseconds of host
// time per call).  A view's maps depend only on its buffers and geometry, the key below.
struct MapKey {
    const void *kd, *vd, *kw, *vw;
    int d, deep_rows, S;
    long long deep_pages, ring_pages;
    bool operator==(const MapKey &o) const {
        return kd == o.kd && vd == o.vd && kw == o.kw && vw == o.vw && d == o.d && deep_rows == o.deep_rows &&
               S == o.S && deep_pages == o.deep_pages && ring_pages == o.ring_pages;
    }
};
struct MapEntry {
    bool used;
    MapKey key;
    CUtensorMap maps[4];  // K deep, V deep, K ring, V ring (the order of RawVerify)
};
constexpr int kMapCache = 8;
MapEntry g_maps[kMapCache];
int g_maps_next = 0;
std::mutex g_maps_mu;

bool cached_maps(const MapKey &k, CUtensorMap *out4) {
    std::lock_guard<std::mutex> lock(g_maps_mu);
    for (int i = 0; i < kMapCache; ++i)
        if (g_maps[i].used && g_maps[i].key == k) {
            std::memcpy(out4, g_maps[i].maps, sizeof(g_maps[i].maps));
            return true;
        }
    return false;
}

void remember_maps(const MapKey &k, const CUtensorMap *in4) {
    std::lock_guard<std::mutex> lock(g_maps_mu);
    MapEntry &e = g_maps[g_maps_next];
    g_maps_next = (g_maps_next + 1) % kMapCache;
    e.used = true;
    e.key = k;
    std::memcpy(e.maps, in4, sizeof(e.maps));
}

}  // namespace

extern "C" int ripe_verify_attn_static(const ripe_cache_view *v, int layer, int r, const void *q, void *out,
                                       float *lse, float scale, uint32_t *device_error, void *stream) {
    using namespace ripe;
    const NvtxRange nvtx_range("ripe_verify_attn_static");
    if (!v || !q || !out) return RIPE_EINVAL;
    const int N = v->batch, L = v->layers, Hq = v->q_heads, kvH = v->kv_heads, d = v->head_dim, R = v->loops;
    if (N < 1 || N > kMaxBatch || L < 1 || Hq < 1 || kvH < 1 || Hq % kvH || (d != 64 && d != 96 && d != 128) ||
        R < 1 || R > kMaxLoops || v->window < 0 || v->max_T < 1 || v->max_B < 1 || v->max_B > kMaxQueryRows ||
        v->max_B > v->max_T || v->max_B * (Hq / kvH) > kMaxQueryRows || v->block_len < 1 ||
        v->block_len > v->max_B ||
        (v->window_mode != RIPE_WINDOW_QUERY_RELATIVE && v->window_mode != RIPE_WINDOW_CACHE_RELATIVE) ||
        layer < 0 || layer >= L || r < 0 || r >= R || !v->k_ring || !v->v_ring || !v->lengths)
        return RIPE_EINVAL;
    const int W = v->window > v->max_T ? v->max_T : v->window;
    const long long s_slots = static_cast<long long>(W) + v->max_B;
    const int S = static_cast<int>(s_slots < v->max_T ? s_slots : v->max_T);
    const int deep_rows = v->max_T - W;
    if (deep_rows > 0 && (!v->k_deep || !v->v_deep)) return RIPE_EINVAL;
    const int g = Hq / kvH;

    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return RIPE_ECUDA;
    DeviceSetup *ds = nullptr;
    const int st = setup_device(dev, ds);
    if (st != RIPE_OK) return st;

    // scratch: partial o, partial (m, l), arrival counters, an error word -- checked against the array
    const int grid = ds->num_sms < 256 ? ds->num_sms : 256;
    const size_t pairs = static_cast<size_t>(N) * kvH;
    const size_t rows = static_cast<size_t>(verify_rows_for(v->block_len * g));
    const size_t slots = static_cast<size_t>(grid) + pairs;
    const size_t off_ml = round256(slots * rows * d * sizeof(float));
    const size_t off_cnt = off_ml + round256(slots * rows * 4 * sizeof(float));
    const size_t off_err = off_cnt + round256(pairs * sizeof(int32_t));
    const size_t need = off_err + 256;
    if (need > RIPE_STATIC_SCRATCH_BYTES) return RIPE_ESCRATCH;

    RawVerify rv;
    std::memset(&rv, 0, sizeof(rv));
    const int deep_box = (deep_rows == 0 || deep_rows >= kTileRows) ? kTileRows : deep_rows;
    const int ring_box = S < kTileRows ? S : kTileRows;
    const long long deep_pages = static_cast<long long>(L) * N * kvH;
    const long long ring_pages = static_cast<long long>(L) * N * R * kvH;
    const MapKey key = {v->k_deep, v->v_deep, v->k_ring, v->v_ring, d, deep_rows, S, deep_pages, ring_pages};
    if (!cached_maps(key, &rv.tmKd)) {
        if (deep_rows > 0 && !(encode(&rv.tmKd, v->k_deep, d, deep_rows, deep_pages, deep_box) &&
                               encode(&rv.tmVd, v->v_deep, d, deep_rows, deep_pages, deep_box)))
            return RIPE_EINVAL;
        if (!encode(&rv.tmKw, v->k_ring, d, S, ring_pages, ring_box) ||
            !encode(&rv.tmVw, v->v_ring, d, S, ring_pages, ring_box))
            return RIPE_EINVAL;
        remember_maps(key, &rv.tmKd);
    }

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned char *base = ds->scratch;
    int32_t *counters = reinterpret_cast<int32_t *>(base + off_cnt);
    uint32_t *err = device_error ? device_error : reinterpret_cast<uint32_t *>(base + off_err);
    // The array keeps the previous call's contents.  The arrival counters need no clearing: each
    // call tags them with its own epoch (never 0 in the low 16 bits), so whatever an earlier call
    // left in them counts as zero.  Our own error word starts each call at zero.
    uint32_t epoch = ds->epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    if ((epoch & 0xFFFFu) == 0) epoch = ds->epoch.fetch_add(1, std::memory_order_relaxed) + 1;
    if (!device_error && cudaMemsetAsync(err, 0, sizeof(uint32_t), s) != cudaSuccess) return RIPE_ECUDA;

    rv.q = q;
    rv.out = out;
    rv.lse = lse;
    rv.T = v->lengths;
    rv.part_o = reinterpret_cast<float *>(base);
    rv.part_ml = reinterpret_cast<float *>(base + off_ml);
    rv.counters = counters;
    rv.epoch = epoch;
    rv.err = err;
    rv.plan.W = W;
    rv.plan.B = v->block_len;
    rv.plan.R = R;
    rv.plan.sink = 0;
    rv.plan.dwin = -1;
    rv.plan.dj = 0;
    rv.plan.nloops = 1;
    rv.plan.loop[0] = static_cast<uint8_t>(r);
    for (int j = 0; j < kMaxQueryRows; ++j) rv.plan.jloop[j] = static_cast<uint8_t>(r);
    rv.plan.ring_slots = S;
    rv.plan.deep_box = deep_box;
    rv.plan.ring_box = ring_box;
    rv.plan.mode_eff = (v->window_mode == RIPE_WINDOW_CACHE_RELATIVE || r == R - 1) ? 1 : 0;
    rv.N = N;
    rv.kvH = kvH;
    rv.g = g;
    rv.Hq = Hq;
    rv.d = d;
    rv.layer = layer;
    rv.grid = grid;
    rv.device = dev;
    rv.num_sms = ds->num_sms;
    rv.dbg_deep_rows = deep_rows;
    rv.dbg_deep_pages = deep_pages;
    rv.dbg_ring_pages = ring_pages;
    rv.has_deep = deep_rows > 0 ? 1 : 0;
    rv.scale = scale;
    const int ls = launch_verify_raw(rv, s);
    if (ls != RIPE_OK) return ls;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}
