// Cache maintenance kernels: append a draft block's plane, accept / roll back with window
// eviction, load a prefix plane, and export the logical view (sm_100a).
//
// RIPE abstract ("Prefix Keys and Values Matter Late: RIPE Caching for Self-Speculative
// Decoding in Looped Language Models", fourth sentence): the deepest plane is stored
// everywhere, all planes only for a window of recent positions.  Layout:
//   deepest region  [L][N][kvH][deep_rows][d]  position t < T - W at row t
//   window ring     [L][N][R][kvH][S][d]       position t >= T - W (and the block) at slot t mod S
// Accept / rollback follows the draft-then-verify scheme of the WaveFront Decoding write-up
// (section on the draft and the check passing through the model at once).
// Every copy moves 16-byte vectors; all kernels are bit-exact data movement.
#include "ripe_common.cuh"

namespace ripe {

__device__ __forceinline__ size_t ring_row(int layer, int n, int plane, int kh, int slot, int N, int R,
                                           int kvH, int S) {
    return (((static_cast<size_t>(layer) * N + n) * R + plane) * kvH + kh) * S + slot;
}

__device__ __forceinline__ size_t deep_row(int layer, int n, int kh, int t, int N, int kvH, int rows) {
    return ((static_cast<size_t>(layer) * N + n) * kvH + kh) * rows + t;
}

// ---------------------------------------------------------------- append
// k, v [N][B][kvH][d] -> ring plane r, slot (T_n + j) mod S.
__global__ void ripe_append_kernel(uint4 *__restrict__ Kw, uint4 *__restrict__ Vw,
                                   const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                   const int32_t *__restrict__ T, uint32_t *err, int N, int B, int kvH,
                                   int d8, int R, int S, int layer, int r, int max_T) {
    // The next launch may start at once: a verify launch reads nothing this kernel writes before
    // its own wait, which returns only after this kernel (and so its predecessor) has completed.
    // Its CTAs then take the SMs that the previous verify launch leaves, while this one waits.
    pdl_trigger();
    pdl_wait();
    const size_t total = static_cast<size_t>(N) * B * kvH * d8;
    for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int c8 = static_cast<int>(idx % d8);
        size_t rest = idx / d8;
        const int kh = static_cast<int>(rest % kvH);
        rest /= kvH;
        const int j = static_cast<int>(rest % B);
        const int n = static_cast<int>(rest / B);
        const int Tn = T[n];
        if (Tn + B > max_T) {
            if (j == 0 && kh == 0 && c8 == 0) atomicOr(err, RIPE_DEVERR_CAPACITY);
            continue;
        }
        const int slot = (Tn + j) % S;
        const size_t dst = ring_row(layer, n, r, kh, slot, N, R, kvH, S) * d8 + c8;
        Kw[dst] = k[idx];
        Vw[dst] = v[idx];
    }
}

int launch_append(ripe_cache *c, int layer, int r, int B, const void *k, const void *v, cudaStream_t s) {
    const int d8 = c->d / 8;
    const size_t total = static_cast<size_t>(c->N) * B * c->kvH * d8;
    int blocks = static_cast<int>((total + 255) / 256);
    if (blocks > 4 * c->num_sms) blocks = 4 * c->num_sms;
    if (blocks < 1) blocks = 1;
    launch_pdl(ripe_append_kernel, dim3(blocks), dim3(256), 0, s, reinterpret_cast<uint4 *>(c->Kw),
               reinterpret_cast<uint4 *>(c->Vw), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
               static_cast<const int32_t *>(c->T_dev), c->err_dev, c->N, B, c->kvH, d8, c->R, c->ring_slots, layer,
               r, c->max_T);
    c->launches += 1;
    c->lengths_dirty = false;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

// ---------------------------------------------------------------- commit / evict
// Accepted length of sequence n: from the host (kernel parameter) or from device memory.
__device__ __forceinline__ int accepted(const HostIntArray &ah, const int32_t *ad, int n, int B,
                                        uint32_t *err, bool report) {
    int a = ad ? ad[n] : ah.v[n];
    if (a < 0 || a > B) {
        if (report) atomicOr(err, RIPE_DEVERR_ACCEPT);
        a = a < 0 ? 0 : B;
    }
    return a;
}

// Positions [max(0, T - W), max(0, T + a - W)) leave the window: their deepest plane moves
// from the ring to the deepest-plane region; planes 0..R-2 are dropped (their slots are
// reused by later positions).  One CTA row per (layer, sequence).
__global__ void ripe_evict_kernel(uint4 *__restrict__ Kd, uint4 *__restrict__ Vd,
                                  const uint4 *__restrict__ Kw, const uint4 *__restrict__ Vw,
                                  const int32_t *__restrict__ T, const HostIntArray acc_h,
                                  const int32_t *acc_d, uint32_t *err, int N, int B, int kvH, int d8,
                                  int R, int S, int W, int deep_rows) {
    pdl_wait();
    pdl_trigger();
    const int layer = blockIdx.x / N;
    const int n = blockIdx.x - layer * N;
    const int Tn = T[n];
    const int a = accepted(acc_h, acc_d, n, B, err, false);
    const int lo = Tn - W > 0 ? Tn - W : 0;
    const int hi = Tn + a - W > 0 ? Tn + a - W : 0;
    const int npos = hi - lo;
    const int work = npos * kvH * d8;
    for (int idx = blockIdx.y * blockDim.x + threadIdx.x; idx < work; idx += gridDim.y * blockDim.x) {
        const int c8 = idx % d8;
        const int rest = idx / d8;
        const int kh = rest % kvH;
        const int t = lo + rest / kvH;
        if (t >= deep_rows) {  // cannot happen while T + B <= max_T
            if (kDebug) atomicOr(err, RIPE_DEVERR_BOUNDS);
            continue;
        }
        const size_t src = ring_row(layer, n, R - 1, kh, t % S, N, R, kvH, S) * d8 + c8;
        const size_t dst = deep_row(layer, n, kh, t, N, kvH, deep_rows) * d8 + c8;
        Kd[dst] = Kw[src];
        Vd[dst] = Vw[src];
    }
}

__global__ void ripe_commit_lengths_kernel(int32_t *T, const HostIntArray acc_h, const int32_t *acc_d,
                                           uint32_t *err, int N, int B) {
    pdl_wait();
    pdl_trigger();
    for (int n = threadIdx.x; n < N; n += blockDim.x) T[n] += accepted(acc_h, acc_d, n, B, err, true);
}

int launch_commit(ripe_cache *c, const int32_t *acc_host, const int32_t *acc_dev, cudaStream_t s) {
    c->lengths_dirty = true;
    HostIntArray ah;
    for (int n = 0; n < c->N; ++n) ah.v[n] = acc_host ? acc_host[n] : 0;
    const int d8 = c->d / 8;
    if (c->deep_rows > 0) {
        const int work = c->B_cur * c->kvH * d8;
        int gy = (work + 255) / 256;
        if (gy < 1) gy = 1;
        dim3 grid(c->L * c->N, gy);
        launch_pdl(ripe_evict_kernel, grid, dim3(256), 0, s, reinterpret_cast<uint4 *>(c->Kd),
                   reinterpret_cast<uint4 *>(c->Vd), reinterpret_cast<const uint4 *>(c->Kw),
                   reinterpret_cast<const uint4 *>(c->Vw), static_cast<const int32_t *>(c->T_dev), ah, acc_dev,
                   c->err_dev, c->N, c->B_cur, c->kvH, d8, c->R, c->ring_slots, c->W, c->deep_rows);
        c->launches += 1;
        if (cudaGetLastError() != cudaSuccess) return RIPE_ECUDA;
    }
    launch_pdl(ripe_commit_lengths_kernel, dim3(1), dim3(256), 0, s, c->T_dev, ah, acc_dev, c->err_dev, c->N,
               c->B_cur);
    c->launches += 1;
    c->lengths_dirty = true;
    if (cudaGetLastError() != cudaSuccess) return RIPE_ECUDA;
    return kDebug ? launch_poison(c, s) : RIPE_OK;
}

// ---------------------------------------------------------------- dead-row poisoning (debug builds)
// After a commit the live rows are: ring slots holding positions [max(0, T - W), T) (every plane)
// and deepest-plane rows [0, max(0, T - W)).  Every other ring slot (rolled-back drafts, positions
// that left the window) and deepest-plane row (not evicted yet) gets the poison pattern, so a kernel
// that reads one with non-zero weight produces a wrong output that the parity tests catch.
__global__ void ripe_poison_kernel(uint4 *__restrict__ Kd, uint4 *__restrict__ Vd, uint4 *__restrict__ Kw,
                                   uint4 *__restrict__ Vw, const int32_t *__restrict__ T, int L, int N, int R,
                                   int kvH, int d8, int S, int W, int deep_rows) {
    const uint32_t pw = kPoisonByte * 0x01010101u;
    const uint4 poison = make_uint4(pw, pw, pw, pw);
    const size_t ring_rows = static_cast<size_t>(L) * N * R * kvH * S;
    const size_t deep_total = static_cast<size_t>(L) * N * kvH * deep_rows;
    const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
    for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < (ring_rows + deep_total) * d8;
         idx += stride) {
        const size_t row = idx / d8;
        if (row < ring_rows) {
            const int slot = static_cast<int>(row % S);
            const size_t rest = row / S / kvH / R;  // layer * N + n
            const int n = static_cast<int>(rest % N);
            const int Tn = T[n];
            const int lo = Tn - W > 0 ? Tn - W : 0;
            const int off = ((slot - lo % S) + S) % S;  // slot of position lo + off
            if (off < Tn - lo) continue;                // a live window position
            Kw[idx] = poison;
            Vw[idx] = poison;
        } else {
            const size_t drow = row - ring_rows;
            const int t = static_cast<int>(drow % deep_rows);
            const int n = static_cast<int>((drow / deep_rows / kvH) % N);
            const int lo = T[n] - W > 0 ? T[n] - W : 0;
            if (t < lo) continue;                       // evicted into the deepest-plane region
            const size_t e = idx - ring_rows * d8;
            Kd[e] = poison;
            Vd[e] = poison;
        }
    }
}

int launch_poison(ripe_cache *c, cudaStream_t s) {
    const int d8 = c->d / 8;
    const size_t rows = static_cast<size_t>(c->L) * c->N * c->kvH * (static_cast<size_t>(c->R) * c->ring_slots +
                                                                      static_cast<size_t>(c->deep_rows));
    size_t blocks = (rows * d8 + 255) / 256;
    if (blocks > static_cast<size_t>(8 * c->num_sms)) blocks = 8 * c->num_sms;
    ripe_poison_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        reinterpret_cast<uint4 *>(c->Kd), reinterpret_cast<uint4 *>(c->Vd), reinterpret_cast<uint4 *>(c->Kw),
        reinterpret_cast<uint4 *>(c->Vw), c->T_dev, c->L, c->N, c->R, c->kvH, d8, c->ring_slots, c->W,
        c->deep_rows);
    c->launches += 1;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

// ---------------------------------------------------------------- prefix load
// One plane of a prefix: plane R-1 of t < T - W goes to the deepest region; positions
// t >= T - W of any plane go to the ring; other planes outside the window are not stored.
__global__ void ripe_load_prefix_kernel(uint4 *__restrict__ Kd, uint4 *__restrict__ Vd, uint4 *__restrict__ Kw,
                                        uint4 *__restrict__ Vw, const uint4 *__restrict__ k,
                                        const uint4 *__restrict__ v, int32_t *T_dev, const HostIntArray Th,
                                        int N, int kvH, int d8, int R, int S, int W, int deep_rows, int layer,
                                        int plane, int Tmax, long long ld_t) {
    if (blockIdx.x == 0)
        for (int n = threadIdx.x; n < N; n += blockDim.x) T_dev[n] = Th.v[n];
    const size_t total = static_cast<size_t>(N) * kvH * Tmax * d8;
    for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int c8 = static_cast<int>(idx % d8);
        size_t rest = idx / d8;
        const int t = static_cast<int>(rest % Tmax);
        rest /= Tmax;
        const int kh = static_cast<int>(rest % kvH);
        const int n = static_cast<int>(rest / kvH);
        const int Tn = Th.v[n];
        if (t >= Tn) continue;
        const size_t src = ((static_cast<size_t>(n) * kvH + kh) * ld_t + t) * d8 + c8;
        if (t < Tn - W) {
            if (plane != R - 1) continue;
            const size_t dst = deep_row(layer, n, kh, t, N, kvH, deep_rows) * d8 + c8;
            Kd[dst] = k[src];
            Vd[dst] = v[src];
        } else {
            const size_t dst = ring_row(layer, n, plane, kh, t % S, N, R, kvH, S) * d8 + c8;
            Kw[dst] = k[src];
            Vw[dst] = v[src];
        }
    }
}

int launch_load_prefix(ripe_cache *c, int layer, int plane, const int32_t *T, const void *k, const void *v,
                       int64_t ld_t, cudaStream_t s) {
    HostIntArray th;
    int Tmax = 0;
    for (int n = 0; n < c->N; ++n) {
        th.v[n] = T[n];
        if (T[n] > Tmax) Tmax = T[n];
    }
    const int d8 = c->d / 8;
    const size_t total = static_cast<size_t>(c->N) * c->kvH * (Tmax > 0 ? Tmax : 1) * d8;
    size_t blocks = (total + 255) / 256;
    if (blocks > static_cast<size_t>(8 * c->num_sms)) blocks = 8 * c->num_sms;
    ripe_load_prefix_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        reinterpret_cast<uint4 *>(c->Kd), reinterpret_cast<uint4 *>(c->Vd), reinterpret_cast<uint4 *>(c->Kw),
        reinterpret_cast<uint4 *>(c->Vw), static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), c->T_dev,
        th, c->N, c->kvH, d8, c->R, c->ring_slots, c->W, c->deep_rows, layer, plane, Tmax > 0 ? Tmax : 1,
        static_cast<long long>(ld_t));
    c->launches += 1;
    c->lengths_dirty = true;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

// ---------------------------------------------------------------- export (test view)
struct PlaneMask {
    uint8_t v[kMaxLoops];
};

__global__ void ripe_export_kernel(const uint4 *__restrict__ Kd, const uint4 *__restrict__ Vd,
                                   const uint4 *__restrict__ Kw, const uint4 *__restrict__ Vw,
                                   const int32_t *__restrict__ T_dev, uint4 *__restrict__ ko, uint4 *__restrict__ vo,
                                   uint8_t *present, const PlaneMask app, int n, int layer, int Tv, int Bcur,
                                   int N, int kvH, int d8, int R, int S, int W, int deep_rows) {
    const int Tn = T_dev[n];
    const size_t total = static_cast<size_t>(R) * kvH * Tv * d8;
    for (size_t idx = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<size_t>(gridDim.x) * blockDim.x) {
        const int c8 = static_cast<int>(idx % d8);
        size_t rest = idx / d8;
        const int t = static_cast<int>(rest % Tv);
        rest /= Tv;
        const int kh = static_cast<int>(rest % kvH);
        const int plane = static_cast<int>(rest / kvH);
        bool pres;
        if (t < Tn) pres = (plane == R - 1) || (t >= Tn - W);
        else pres = (t < Tn + Bcur) && app.v[plane];
        uint4 kx = make_uint4(0, 0, 0, 0), vx = make_uint4(0, 0, 0, 0);
        if (pres) {
            size_t src;
            if (t < Tn - W) {
                src = deep_row(layer, n, kh, t, N, kvH, deep_rows) * d8 + c8;
                kx = Kd[src];
                vx = Vd[src];
            } else {
                src = ring_row(layer, n, plane, kh, t % S, N, R, kvH, S) * d8 + c8;
                kx = Kw[src];
                vx = Vw[src];
            }
        }
        ko[idx] = kx;
        vo[idx] = vx;
        if (kh == 0 && c8 == 0) present[static_cast<size_t>(plane) * Tv + t] = pres ? 1 : 0;
    }
}

int launch_export(ripe_cache *c, int n, int layer, void *k_out, void *v_out, uint8_t *present, cudaStream_t s) {
    PlaneMask app;
    for (int p = 0; p < kMaxLoops; ++p) app.v[p] = (p < c->R) ? c->appended[layer * c->R + p] : 0;
    const int Tv = c->T[n] + c->B_cur;
    if (Tv == 0) return RIPE_OK;
    const int d8 = c->d / 8;
    const size_t total = static_cast<size_t>(c->R) * c->kvH * Tv * d8;
    size_t blocks = (total + 255) / 256;
    if (blocks > static_cast<size_t>(8 * c->num_sms)) blocks = 8 * c->num_sms;
    ripe_export_kernel<<<static_cast<int>(blocks), 256, 0, s>>>(
        reinterpret_cast<const uint4 *>(c->Kd), reinterpret_cast<const uint4 *>(c->Vd),
        reinterpret_cast<const uint4 *>(c->Kw), reinterpret_cast<const uint4 *>(c->Vw), c->T_dev,
        static_cast<uint4 *>(k_out), static_cast<uint4 *>(v_out), present, app, n, layer, Tv, c->B_cur, c->N,
        c->kvH, d8, c->R, c->ring_slots, c->W, c->deep_rows);
    c->launches += 1;
    return cudaGetLastError() == cudaSuccess ? RIPE_OK : RIPE_ECUDA;
}

}  // namespace ripe
