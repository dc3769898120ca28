// Host side of the C ABI declared in include/ripe.h: argument and state validation,
// allocation of the cache regions, TMA descriptors, and the host copy of the state.
#include <algorithm>
#include <cstdlib>
#include <cstring>
#include <new>

#include "ripe_common.cuh"

using namespace ripe;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 3-D bf16 map over [pages][rows][d]: box = 32 elements (64 bytes, 64-byte swizzle) x box_rows x 1.
bool encode_map(CUtensorMap *m, void *base, int d, int rows, long long pages, int box_rows) {
    EncodeTiledFn enc = get_encoder();
    if (!enc) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(pages)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * 2 * rows};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(kBoxCols), static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

void release(ripe_cache *c) {
    if (!c) return;
    cudaFree(c->Kd);
    cudaFree(c->Vd);
    cudaFree(c->Kw);
    cudaFree(c->Vw);
    cudaFree(c->T_dev);
    cudaFree(c->err_dev);
    cudaFree(c->part_o);
    cudaFree(c->part_ml);
    cudaFree(c->counters);
    delete c;
}

template <typename T>
bool dalloc(T **p, size_t bytes, int64_t *acct, int fill = 0) {
    *p = nullptr;
    if (bytes == 0) return true;
    if (cudaMalloc(reinterpret_cast<void **>(p), bytes) != cudaSuccess) {
        *p = nullptr;
        cudaGetLastError();
        return false;
    }
    *acct += static_cast<int64_t>(bytes);
    return cudaMemset(*p, fill, bytes) == cudaSuccess;
}

// Calls run with the cache's device current.
struct DeviceGuard {
    int prev = -1;
    bool ok = true;
    explicit DeviceGuard(int dev) {
        if (cudaGetDevice(&prev) != cudaSuccess) { ok = false; return; }
        if (prev != dev && cudaSetDevice(dev) != cudaSuccess) ok = false;
    }
    ~DeviceGuard() {
        int cur;
        if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
    }
};

bool any_drafted(const ripe_cache *c) {
    for (size_t i = 0; i < c->drafted.size(); ++i)
        if (c->drafted[i]) return true;
    return false;
}

bool all_appended(const ripe_cache *c) {
    for (size_t i = 0; i < c->appended.size(); ++i)
        if (!c->appended[i]) return false;
    return true;
}

}  // namespace

extern "C" {

const char *ripe_strerror(int status) {
    switch (status) {
        case RIPE_OK: return "ok";
        case RIPE_EINVAL: return "invalid argument";
        case RIPE_ENOMEM: return "out of memory";
        case RIPE_ECAPACITY: return "cache capacity exceeded";
        case RIPE_ESTATE: return "call out of order for the cache state";
        case RIPE_ECUDA: return "CUDA error";
        case RIPE_ESCRATCH: return "problem exceeds the static scratch of ripe_verify_attn_static";
        default: return "unknown status";
    }
}

int ripe_cache_alloc(int batch, int layers, int q_heads, int kv_heads, int head_dim, int loops, int window,
                     int max_T, int max_B, int window_mode, ripe_cache_t **out) {
    const NvtxRange nvtx_range("ripe_cache_alloc");
    if (!out) return RIPE_EINVAL;
    *out = nullptr;
    if (batch < 1 || batch > kMaxBatch || layers < 1 || q_heads < 1 || kv_heads < 1 || q_heads % kv_heads ||
        (head_dim != 64 && head_dim != 96 && head_dim != 128) || loops < 1 || loops > kMaxLoops || window < 0 ||
        max_T < 1 || max_B < 1 || max_B > kMaxQueryRows || max_B > max_T ||
        max_B * (q_heads / kv_heads) > kMaxQueryRows ||
        (window_mode != RIPE_WINDOW_QUERY_RELATIVE && window_mode != RIPE_WINDOW_CACHE_RELATIVE))
        return RIPE_EINVAL;

    ripe_cache *c = new (std::nothrow) ripe_cache();
    if (!c) return RIPE_ENOMEM;
    c->N = batch; c->L = layers; c->Hq = q_heads; c->kvH = kv_heads; c->g = q_heads / kv_heads;
    c->d = head_dim; c->R = loops; c->max_T = max_T; c->max_B = max_B; c->mode = window_mode;
    c->W = window > max_T ? max_T : window;  // a window of max_T already keeps every plane
    const long long s_slots = static_cast<long long>(c->W) + max_B;
    c->ring_slots = static_cast<int>(s_slots < max_T ? s_slots : max_T);
    c->deep_rows = max_T - c->W;
    c->deep_box = (c->deep_rows == 0 || c->deep_rows >= kTileRows) ? kTileRows : c->deep_rows;
    c->ring_box = c->ring_slots < kTileRows ? c->ring_slots : kTileRows;
    c->T.assign(batch, 0);
    c->B_cur = 0;
    c->appended.assign(static_cast<size_t>(layers) * loops, 0);
    c->drafted.assign(static_cast<size_t>(layers) * loops, 0);
    c->prefix_set = false;
    c->synced = true;
    c->lengths_dirty = true;
    c->kv_bytes = c->scratch_bytes = 0;
    c->launches = 0;

    if (cudaGetDevice(&c->device) != cudaSuccess || c->device >= kMaxDevices ||
        cudaDeviceGetAttribute(&c->num_sms, cudaDevAttrMultiProcessorCount, c->device) != cudaSuccess) {
        cudaGetLastError();
        delete c;
        return RIPE_ECUDA;
    }
    const size_t d = head_dim;
    const size_t deep_elems = static_cast<size_t>(layers) * batch * kv_heads * c->deep_rows * d;
    const size_t ring_elems = static_cast<size_t>(layers) * batch * loops * kv_heads * c->ring_slots * d;
    c->part_rows = 16 * cdiv(max_B * c->g, 16);
    if (c->part_rows > 16 && c->part_rows < 32) c->part_rows = 32;
    if (c->part_rows > 32) c->part_rows = 64;
    c->part_slots = c->num_sms + batch * kv_heads;
    const int kv_fill = kDebug ? kPoisonByte : 0;  // debug builds: no row holds a position yet
    bool ok = dalloc(&c->Kd, deep_elems * 2, &c->kv_bytes, kv_fill) &&
              dalloc(&c->Vd, deep_elems * 2, &c->kv_bytes, kv_fill) &&
              dalloc(&c->Kw, ring_elems * 2, &c->kv_bytes, kv_fill) &&
              dalloc(&c->Vw, ring_elems * 2, &c->kv_bytes, kv_fill) &&
              dalloc(&c->T_dev, batch * sizeof(int32_t), &c->scratch_bytes) &&
              dalloc(&c->err_dev, sizeof(uint32_t), &c->scratch_bytes) &&
              dalloc(&c->part_o, static_cast<size_t>(c->part_slots) * c->part_rows * d * sizeof(float),
                     &c->scratch_bytes) &&
              dalloc(&c->part_ml, static_cast<size_t>(c->part_slots) * c->part_rows * 4 * sizeof(float),
                     &c->scratch_bytes) &&
              dalloc(&c->counters, static_cast<size_t>(batch) * kv_heads * sizeof(int32_t), &c->scratch_bytes);
    if (!ok) {
        release(c);
        return RIPE_ENOMEM;
    }
    std::memset(&c->tm_Kd, 0, sizeof(CUtensorMap));
    std::memset(&c->tm_Vd, 0, sizeof(CUtensorMap));
    const long long deep_pages = static_cast<long long>(layers) * batch * kv_heads;
    const long long ring_pages = static_cast<long long>(layers) * batch * loops * kv_heads;
    if (c->deep_rows > 0) {
        ok = encode_map(&c->tm_Kd, c->Kd, head_dim, c->deep_rows, deep_pages, c->deep_box) &&
             encode_map(&c->tm_Vd, c->Vd, head_dim, c->deep_rows, deep_pages, c->deep_box);
    }
    ok = ok && encode_map(&c->tm_Kw, c->Kw, head_dim, c->ring_slots, ring_pages, c->ring_box) &&
         encode_map(&c->tm_Vw, c->Vw, head_dim, c->ring_slots, ring_pages, c->ring_box);
    if (!ok || ensure_verify_attributes(c->device) != RIPE_OK || cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        release(c);
        return RIPE_ECUDA;
    }
    *out = c;
    return RIPE_OK;
}

int ripe_cache_free(ripe_cache_t *c) {
    const NvtxRange nvtx_range("ripe_cache_free");
    if (!c) return RIPE_OK;
    DeviceGuard g(c->device);
    cudaDeviceSynchronize();
    release(c);
    return RIPE_OK;
}

int ripe_load_prefix(ripe_cache_t *c, int layer, int plane, const int32_t *T, const void *k, const void *v,
                     int64_t ld_t, void *stream) {
    const NvtxRange nvtx_range("ripe_load_prefix");
    if (!c || !T || !k || !v || layer < 0 || layer >= c->L || plane < 0 || plane >= c->R) return RIPE_EINVAL;
    if (c->B_cur != 0 || !c->synced || any_drafted(c)) return RIPE_ESTATE;
    int Tmax = 0;
    for (int n = 0; n < c->N; ++n) {
        if (T[n] < 0) return RIPE_EINVAL;
        if (T[n] + 1 > c->max_T) return RIPE_ECAPACITY;
        if (T[n] > Tmax) Tmax = T[n];
    }
    if (ld_t < Tmax || ld_t < 1) return RIPE_EINVAL;
    if (c->prefix_set)
        for (int n = 0; n < c->N; ++n)
            if (T[n] != c->T[n]) return RIPE_EINVAL;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int st = launch_load_prefix(c, layer, plane, T, k, v, ld_t, static_cast<cudaStream_t>(stream));
    if (st != RIPE_OK) return st;
    for (int n = 0; n < c->N; ++n) c->T[n] = T[n];
    c->prefix_set = true;
    return RIPE_OK;
}

int ripe_append_block(ripe_cache_t *c, int layer, int r, int B, const void *k, const void *v, void *stream) {
    const NvtxRange nvtx_range("ripe_append_block");
    if (!c || !k || !v || layer < 0 || layer >= c->L || r < 0 || r >= c->R || B < 1 || B > c->max_B)
        return RIPE_EINVAL;
    if (c->B_cur != 0 && B != c->B_cur) return RIPE_EINVAL;
    for (int n = 0; n < c->N; ++n)
        if (c->T[n] + B > c->max_T) return RIPE_ECAPACITY;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int st = launch_append(c, layer, r, B, k, v, static_cast<cudaStream_t>(stream));
    if (st != RIPE_OK) return st;
    c->B_cur = B;
    c->appended[static_cast<size_t>(layer) * c->R + r] = 1;
    c->prefix_set = true;
    return RIPE_OK;
}

int ripe_verify_attn(ripe_cache_t *c, int layer, int r, const void *q, void *out, float *lse, float scale,
                     void *stream) {
    const NvtxRange nvtx_range("ripe_verify_attn");
    if (!c || !q || !out || layer < 0 || layer >= c->L || r < 0 || r >= c->R) return RIPE_EINVAL;
    if (c->B_cur == 0 || !c->appended[static_cast<size_t>(layer) * c->R + r]) return RIPE_ESTATE;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    return launch_verify(c, layer, r, q, out, lse, scale, static_cast<cudaStream_t>(stream));
}

int ripe_append_verify(ripe_cache_t *c, int layer, int r, int B, const void *k, const void *v, const void *q,
                       void *out, float *lse, float scale, void *stream) {
    const NvtxRange nvtx_range("ripe_append_verify");
    if (!c || !k || !v || !q || !out || layer < 0 || layer >= c->L || r < 0 || r >= c->R || B < 1 ||
        B > c->max_B)
        return RIPE_EINVAL;
    if (c->B_cur != 0 && B != c->B_cur) return RIPE_EINVAL;
    for (int n = 0; n < c->N; ++n)
        if (c->T[n] + B > c->max_T) return RIPE_ECAPACITY;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int prev_B = c->B_cur;
    c->B_cur = B;  // the kernel plans the block's tiles with this length
    const int st = launch_verify(c, layer, r, q, out, lse, scale, static_cast<cudaStream_t>(stream), k, v);
    if (st != RIPE_OK) {
        c->B_cur = prev_B;
        return st;
    }
    c->appended[static_cast<size_t>(layer) * c->R + r] = 1;
    c->prefix_set = true;
    return RIPE_OK;
}

static int draft_step(ripe_cache_t *c, int layer, int r, int j, int sink, int window, const void *k, const void *v,
                      const void *q, void *out, float *lse, float scale, void *stream) {
    if (!c || !k || !v || !q || !out || layer < 0 || layer >= c->L || r < 0 || r >= c->R || j < 0 ||
        j >= c->max_B)
        return RIPE_EINVAL;
    const size_t idx = static_cast<size_t>(layer) * c->R + r;
    if (c->B_cur != 0 || j > c->drafted[idx]) return RIPE_ESTATE;
    for (int n = 0; n < c->N; ++n)
        if (c->T[n] + j + 1 > c->max_T) return RIPE_ECAPACITY;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int st = launch_draft(c, layer, r, j, k, v, q, out, lse, scale, static_cast<cudaStream_t>(stream), sink,
                                window);
    if (st != RIPE_OK) return st;
    c->drafted[idx] = j + 1;  // a later position of this plane is stale once j is redrafted
    c->prefix_set = true;
    return RIPE_OK;
}

int ripe_draft_attn(ripe_cache_t *c, int layer, int r, int j, const void *k, const void *v, const void *q,
                    void *out, float *lse, float scale, void *stream) {
    const NvtxRange nvtx_range("ripe_draft_attn");
    return draft_step(c, layer, r, j, 0, -1, k, v, q, out, lse, scale, stream);
}

int ripe_draft_attn_window(ripe_cache_t *c, int layer, int r, int j, int sink, int window, const void *k,
                           const void *v, const void *q, void *out, float *lse, float scale, void *stream) {
    const NvtxRange nvtx_range("ripe_draft_attn_window");
    if (sink < 0 || window < 0) return RIPE_EINVAL;
    return draft_step(c, layer, r, j, sink, window, k, v, q, out, lse, scale, stream);
}

int ripe_verify_attn_wave(ripe_cache_t *c, int layer, const int32_t *loop_of_position, const void *q, void *out,
                          float *lse, float scale, void *stream) {
    const NvtxRange nvtx_range("ripe_verify_attn_wave");
    if (!c || !loop_of_position || !q || !out || layer < 0 || layer >= c->L) return RIPE_EINVAL;
    if (c->B_cur == 0) return RIPE_ESTATE;
    for (int j = 0; j < c->B_cur; ++j) {
        const int r = loop_of_position[j];
        if (r < 0 || r >= c->R) return RIPE_EINVAL;
        if (!c->appended[static_cast<size_t>(layer) * c->R + r]) return RIPE_ESTATE;
    }
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    return launch_verify_wave(c, layer, loop_of_position, q, out, lse, scale, static_cast<cudaStream_t>(stream));
}

int ripe_commit(ripe_cache_t *c, const int32_t *accepted_len, void *stream) {
    const NvtxRange nvtx_range("ripe_commit");
    if (!c || !accepted_len) return RIPE_EINVAL;
    if (c->B_cur == 0 || !all_appended(c)) return RIPE_ESTATE;
    for (int n = 0; n < c->N; ++n)
        if (accepted_len[n] < 0 || accepted_len[n] > c->B_cur) return RIPE_EINVAL;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int st = launch_commit(c, accepted_len, nullptr, static_cast<cudaStream_t>(stream));
    if (st != RIPE_OK) return st;
    for (int n = 0; n < c->N; ++n) c->T[n] += accepted_len[n];
    c->B_cur = 0;
    std::fill(c->appended.begin(), c->appended.end(), 0);
    std::fill(c->drafted.begin(), c->drafted.end(), 0);
    return RIPE_OK;
}

int ripe_commit_device(ripe_cache_t *c, const int32_t *accepted_len, void *stream) {
    const NvtxRange nvtx_range("ripe_commit_device");
    if (!c || !accepted_len) return RIPE_EINVAL;
    if (c->B_cur == 0 || !all_appended(c)) return RIPE_ESTATE;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    const int st = launch_commit(c, nullptr, accepted_len, static_cast<cudaStream_t>(stream));
    if (st != RIPE_OK) return st;
    for (int n = 0; n < c->N; ++n) c->T[n] += c->B_cur;  // upper bound until synced
    c->synced = false;
    c->B_cur = 0;
    std::fill(c->appended.begin(), c->appended.end(), 0);
    std::fill(c->drafted.begin(), c->drafted.end(), 0);
    return RIPE_OK;
}

int ripe_sync_lengths(ripe_cache_t *c, int32_t *T_out, void *stream) {
    const NvtxRange nvtx_range("ripe_sync_lengths");
    if (!c) return RIPE_EINVAL;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(c->T.data(), c->T_dev, c->N * sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return RIPE_ECUDA;
    c->synced = true;
    if (T_out) std::memcpy(T_out, c->T.data(), c->N * sizeof(int32_t));
    return RIPE_OK;
}

int ripe_cache_stats(const ripe_cache_t *c, ripe_stats *st) {
    if (!c || !st) return RIPE_EINVAL;
    int64_t stored = 0, full = 0;
    for (int n = 0; n < c->N; ++n) {
        const int64_t T = c->T[n];
        stored += T + (T < c->W ? T : c->W) * (c->R - 1);
        full += T * c->R;
    }
    st->stored_position_planes = stored;
    st->full_position_planes = full;
    st->kv_bytes = c->kv_bytes;
    st->scratch_bytes = c->scratch_bytes;
    st->deep_rows = c->deep_rows;
    st->ring_slots = c->ring_slots;
    st->block_len = c->B_cur;
    st->lengths_synced = c->synced ? 1 : 0;
    return RIPE_OK;
}

int ripe_cache_export(ripe_cache_t *c, int n, int layer, void *k_out, void *v_out, uint8_t *plane_present,
                      void *stream) {
    const NvtxRange nvtx_range("ripe_cache_export");
    if (!c || !k_out || !v_out || !plane_present || n < 0 || n >= c->N || layer < 0 || layer >= c->L)
        return RIPE_EINVAL;
    if (!c->synced) return RIPE_ESTATE;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    return launch_export(c, n, layer, k_out, v_out, plane_present, static_cast<cudaStream_t>(stream));
}

int ripe_get_device_error(ripe_cache_t *c, uint32_t *err_out, void *stream) {
    const NvtxRange nvtx_range("ripe_get_device_error");
    if (!c || !err_out) return RIPE_EINVAL;
    DeviceGuard g(c->device);
    if (!g.ok) return RIPE_ECUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t e = 0;
    if (cudaMemcpyAsync(&e, c->err_dev, sizeof(e), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return RIPE_ECUDA;
    *err_out = e;
    if (e) {  // a kernel stopped early: clear the word and the merge counters it may have left
        if (cudaMemsetAsync(c->err_dev, 0, sizeof(uint32_t), s) != cudaSuccess ||
            cudaMemsetAsync(c->counters, 0, static_cast<size_t>(c->N) * c->kvH * sizeof(int32_t), s) !=
                cudaSuccess ||
            cudaStreamSynchronize(s) != cudaSuccess)
            return RIPE_ECUDA;
    }
    return RIPE_OK;
}

int64_t ripe_launch_count(const ripe_cache_t *c) { return c ? c->launches : -1; }

int ripe_build_info(void) { return kDebug ? RIPE_BUILD_DEBUG : 0; }

int ripe_set_verify_consumer(int consumer) { return ripe::set_verify_consumer(consumer); }

int ripe_get_verify_consumer(void) { return ripe::get_verify_consumer(); }

}  // extern "C"
