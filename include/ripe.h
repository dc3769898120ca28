/*
 * ripe.h -- C ABI of the RIPE verify-attention library (libripe.so, sm_100a).
 *
 * A looped language model runs one block of layers R times per token, so each
 * recurrent layer has R planes of keys and values per position; the verify
 * pass of self-speculative decoding reads them at every loop r.  RIPE keeps
 * the deepest plane (r = R-1) of every position and all R planes only for a
 * window of the W most recent positions.
 *   Source: "Prefix Keys and Values Matter Late: RIPE Caching for
 *   Self-Speculative Decoding in Looped Language Models" (arXiv 2610.34436),
 *   abstract, first, fourth and fifth sentences.
 * Accept / rollback of a draft block follows the draft-then-verify scheme as
 * described in the WaveFront Decoding write-up (rit.work blog, the section on
 * drafting and checking in one pass): the verified prefix of the block is kept,
 * the full-depth token replaces the first mismatch, and the drafts after it are
 * discarded.
 *
 * Conventions for every call:
 *   - Device pointers are plain CUDA device addresses owned by the caller and
 *     must stay valid until the work enqueued on `stream` has finished.
 *     Host pointers are read before the call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All device
 *     work is enqueued on it; calls return after enqueueing.
 *   - bf16 tensors are IEEE bfloat16, contiguous, row-major in the order given.
 *   - Argument and state errors are detected on the host before anything is
 *     enqueued and leave the cache unchanged.  A failed launch returns
 *     RIPE_ECUDA.  Faults detected by a kernel (a wait that gave up, a block
 *     that would overflow the capacity) set bits in a device error word read
 *     by ripe_get_device_error(); kernels never trap.
 *   - A cache handle is not thread-safe and must be used from one stream at a
 *     time: calls on one handle share scratch memory on the device.
 */
#ifndef RIPE_H
#define RIPE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ripe_cache ripe_cache_t;

/* Status codes returned by every call. */
enum ripe_status {
    RIPE_OK = 0,
    RIPE_EINVAL = -1,    /* bad argument (shape, index, null pointer, unsupported size) */
    RIPE_ENOMEM = -2,    /* device or host allocation failed */
    RIPE_ECAPACITY = -3, /* committed + block positions would exceed max_T */
    RIPE_ESTATE = -4,    /* call out of order (e.g. verify before the plane was appended) */
    RIPE_ECUDA = -5,     /* a CUDA runtime call or kernel launch failed */
    RIPE_ESCRATCH = -6   /* the allocation-free entry point's static scratch is too small */
};

/* How the window of full-depth positions is measured for a query at position p = T + j.
 * QUERY_RELATIVE (default): key t reads plane r when t >= p - W; this is the rule under
 *   which a window at least as long as the draft block makes batched verification
 *   independent of how positions are split into blocks (RIPE abstract, fifth sentence).
 * CACHE_RELATIVE: key t reads plane r when t >= T - W for every query of the block.
 * In both modes the draft block's own keys read plane r (their deeper planes do not exist
 * yet) and every other key reads the deepest plane R-1. */
enum ripe_window_mode { RIPE_WINDOW_QUERY_RELATIVE = 0, RIPE_WINDOW_CACHE_RELATIVE = 1 };

/* Device error bits reported by ripe_get_device_error(). */
enum ripe_device_error {
    RIPE_DEVERR_WAIT_TIMEOUT = 1u, /* a kernel gave up waiting for its own copies */
    RIPE_DEVERR_CAPACITY = 2u,     /* a kernel saw T + B > max_T and skipped its work */
    RIPE_DEVERR_ACCEPT = 4u,       /* a device-side accepted length was outside [0, B] */
    RIPE_DEVERR_BOUNDS = 8u        /* debug builds: a tile, slot or scratch index fell outside its
                                      region (the access is still made in bounds: TMA clips it) */
};

/* Bits of ripe_build_info(). */
enum ripe_build_flags {
    RIPE_BUILD_DEBUG = 1 /* built with -DRIPE_DEBUG: device-side index checks set RIPE_DEVERR_BOUNDS,
                            and every commit fills the ring slots and deepest-plane rows that hold
                            no live position with the largest finite bf16 (0x7F7F), so that a read
                            of a dead slot with non-zero weight shows up as a wrong (huge or
                            non-finite) output instead of a plausible stale value */
};

typedef struct ripe_stats {
    int64_t stored_position_planes; /* sum over sequences of (position, plane) pairs kept for
                                       the committed positions, per layer and key/value head:
                                       T_n + min(W, T_n) * (R - 1) per sequence */
    int64_t full_position_planes;   /* the same for the full cache: R * T_n per sequence */
    int64_t kv_bytes;               /* device bytes of the key/value regions (all layers) */
    int64_t scratch_bytes;          /* device bytes of per-call scratch and metadata */
    int32_t deep_rows;              /* rows per (layer, sequence, kv head) of the deepest-plane region */
    int32_t ring_slots;             /* slots per (layer, sequence, plane, kv head) of the window ring */
    int32_t block_len;              /* B of the draft block in flight, 0 when none */
    int32_t lengths_synced;         /* 1 when the host copy of T_n is current */
} ripe_stats;

/*
 * Allocate a cache for `batch` sequences (1 .. 1024: the verify kernels keep every sequence's
 * length and tile count in shared memory).
 *   layers      recurrent layers L (>= 1)
 *   q_heads     query heads Hq; kv_heads divides it, query head h uses kv head h / (Hq / kv_heads)
 *   head_dim    d, one of 64, 96, 128
 *   loops       R (1 .. 256); plane R-1 is the deepest
 *   window      W >= 0; W >= max_T stores every plane (full cache), W = 0 keeps only the deepest
 *   max_T       capacity per sequence: committed positions + draft block <= max_T
 *   max_B       largest draft block (1 .. 64, and max_B * Hq / kv_heads <= 64)
 *   window_mode enum ripe_window_mode
 * Device layout (bf16):
 *   deepest plane  K,V [L][batch][kv_heads][max(0, max_T - W)][d]   position t at row t
 *   window ring    K,V [L][batch][R][kv_heads][S][d], S = min(W + max_B, max_T),
 *                  position t at slot t mod S
 * The library owns all cache memory and frees it in ripe_cache_free().  Every cache starts
 * empty (T_n = 0).  On failure *out is NULL.
 */
int ripe_cache_alloc(int batch, int layers, int q_heads, int kv_heads, int head_dim, int loops,
                     int window, int max_T, int max_B, int window_mode, ripe_cache_t **out);

/* Free a cache and its device memory (synchronises the device first).  NULL is a no-op. */
int ripe_cache_free(ripe_cache_t *c);

/*
 * Load one plane of a prefix for one layer (RIPE abstract, fourth sentence: the deepest
 * plane is kept everywhere, the other planes only inside the window).
 *   T       host int32[batch], committed prefix length of each sequence; the first load
 *           sets the lengths, later loads (other layers or planes) must pass the same values
 *   plane   0 .. R-1
 *   k, v    device bf16 [batch][kv_heads][ld_t][d], positions 0 .. T_n - 1 of this plane
 *   ld_t    row stride in positions, >= max over n of T_n
 * Plane R-1 is stored for every position; other planes only for positions t >= T_n - W.
 * Requires no draft block in flight (RIPE_ESTATE) and T_n + 1 <= max_T (RIPE_ECAPACITY).
 */
int ripe_load_prefix(ripe_cache_t *c, int layer, int plane, const int32_t *T, const void *k,
                     const void *v, int64_t ld_t, void *stream);

/*
 * Append plane r of the current draft block of one layer: block position j of sequence n
 * (absolute position T_n + j) goes to ring slot (T_n + j) mod S of plane r.
 *   B      block length, 1 .. max_B; all appends of one block use the same B
 *   k, v   device bf16 [batch][B][kv_heads][d]
 * The block's planes are computed while it is verified (RIPE abstract, first sentence:
 * verification runs all R loops), so plane r must be appended before ripe_verify_attn(.., r).
 * Errors: RIPE_ECAPACITY if T_n + B > max_T for some n.
 */
int ripe_append_block(ripe_cache_t *c, int layer, int r, int B, const void *k, const void *v,
                      void *stream);

/*
 * Verification attention of the draft block at loop r for one layer.
 * For query head h of block position j of sequence n (p = T_n + j) and every key t <= p:
 * the key/value plane is r when t >= T_n (draft block) or t is inside the window (see
 * enum ripe_window_mode), else the deepest plane R-1; out is the causal softmax attention
 * softmax_t(scale * <q, K_plane[t]>) . V_plane[t].
 *   q      device bf16 [batch][B][q_heads][d]
 *   out    device bf16 [batch][B][q_heads][d], rounded to nearest even from fp32
 *   lse    device fp32 [batch][B][q_heads] natural-log softmax normaliser, or NULL
 *   scale  logit scale (1/sqrt(d) for unscaled queries)
 * Requires plane r of the block appended for this layer (else RIPE_ESTATE).
 * Work: split-KV over the deepest-plane region and the window ring in one persistent
 * launch; partial results are merged in the same launch, through the shared memory of a
 * 2-CTA cluster when two CTAs share a (sequence, kv head), else through per-call scratch
 * owned by the cache.  The contractions run on tensor cores: mma.sync tiles, or for 9..64 query
 * rows per kv head the tcgen05 consumer when ripe_set_verify_consumer selects it.
 */
int ripe_verify_attn(ripe_cache_t *c, int layer, int r, const void *q, void *out, float *lse,
                     float scale, void *stream);

/*
 * ripe_append_block(c, layer, r, B, k, v) followed by ripe_verify_attn(c, layer, r, q, ...) in
 * one launch: plane r of the draft block is written into the window ring by the verify kernel
 * itself, just before the one tile of this launch that reads those rows.  Arguments, layouts,
 * results and errors are those of the two calls; the result is identical.
 */
int ripe_append_verify(ripe_cache_t *c, int layer, int r, int B, const void *k, const void *v,
                       const void *q, void *out, float *lse, float scale, void *stream);

/*
 * One step of the draft phase: block position j at loop r, written and attended in one launch.
 * Draft-then-verify builds the draft block one position at a time at a shallow depth, then
 * checks the whole block at full depth (RIPE abstract, first sentence; WaveFront write-up,
 * section on drafting and checking in one pass).  Plane r of position T_n + j is written to
 * ring slot (T_n + j) mod S from k, v; then the query of that position attends over keys
 * t <= T_n + j with the plane rule of ripe_verify_attn for query p = T_n + j: the draft
 * positions 0 .. j at plane r, the window at plane r, older keys at the deepest plane.
 * The result equals row j of ripe_verify_attn over a block whose plane r holds the same rows.
 *   j        0 .. max_B - 1; positions 0 .. j-1 of plane r must have been drafted since the
 *            last commit (else RIPE_ESTATE); redrafting j makes later drafted positions stale
 *   k, v     device bf16 [batch][1][kv_heads][d], plane r of position j
 *   q, out   device bf16 [batch][1][q_heads][d];  lse  device fp32 [batch][1][q_heads] or NULL
 * Requires no verification block in flight (the first ripe_append_block of the block ends the
 * draft phase; RIPE_ESTATE) and T_n + j + 1 <= max_T (RIPE_ECAPACITY).  ripe_commit (or
 * ripe_commit_device) ends the draft phase of the block; ripe_load_prefix is refused while a
 * draft is in flight.
 */
int ripe_draft_attn(ripe_cache_t *c, int layer, int r, int j, const void *k, const void *v,
                    const void *q, void *out, float *lse, float scale, void *stream);

/*
 * ripe_draft_attn with windowed draft attention: a sliding window plus an attention sink on
 * the draft's attention only, verification untouched ("Windowed-MTP: Removing the
 * Full-Context Draft-KV Tax at Million-Token Context", abstract).  The query of position
 * p = T_n + j attends only to the keys t <= p with t < sink or t >= p - window, each read at
 * the plane the rule of ripe_verify_attn gives it; the deepest-plane keys in between are not
 * read, so the draft's read is bounded by sink + window + W + B positions whatever T_n is.
 *   sink    >= 0 positions at the start of the sequence always attended
 *   window  >= 0; window >= T_n + j attends every key (the same result as ripe_draft_attn)
 * Other arguments, state rules and errors as for ripe_draft_attn.
 */
int ripe_draft_attn_window(ripe_cache_t *c, int layer, int r, int j, int sink, int window, const void *k,
                           const void *v, const void *q, void *out, float *lse, float scale, void *stream);

/*
 * Verification attention with a loop per block position: block position j is evaluated
 * exactly as ripe_verify_attn(.., loop_of_position[j], ..) would evaluate it.  This is the
 * shape of a wavefront schedule, where one batched pass of the looped block holds positions
 * at different depths (WaveFront write-up, sections on drafting and checking in one pass and on
 * the long-context bottleneck: positions at different depths read different KV regions).
 * The deepest-plane region is read once for all positions; the window ring once per distinct
 * loop.  With RIPE this reads T + n_loops * (W + B) key rows per (sequence, kv head), where a
 * full cache reads n_loops * (T + B).
 *   loop_of_position  host int32[B], each 0 .. R-1 with that plane of the block appended
 *   q, out, lse, scale as for ripe_verify_attn
 */
int ripe_verify_attn_wave(ripe_cache_t *c, int layer, const int32_t *loop_of_position, const void *q,
                          void *out, float *lse, float scale, void *stream);

/*
 * Accept a prefix of the draft block of every sequence and roll back the rest
 * (WaveFront write-up, draft-then-verify): accepted_len[n] in 0 .. B positions of the block
 * become committed, T_n += accepted_len[n]; the other block positions are discarded.
 * Positions that leave the window (t < T_n - W) move their deepest plane from the ring into
 * the deepest-plane region, and planes 0 .. R-2 of them are dropped (RIPE abstract, fourth
 * sentence).  Requires every plane of the block appended for every layer (RIPE_ESTATE).
 *   accepted_len  host int32[batch]
 */
int ripe_commit(ripe_cache_t *c, const int32_t *accepted_len, void *stream);

/*
 * Same as ripe_commit with the accepted lengths in device memory (device int32[batch]), for
 * decoders that compute acceptance on the GPU.  Values outside 0 .. B are clamped and set
 * RIPE_DEVERR_ACCEPT.  The host copy of T_n becomes stale until ripe_sync_lengths(); until
 * then host-side capacity checks assume every device commit accepted the whole block.
 */
int ripe_commit_device(ripe_cache_t *c, const int32_t *accepted_len, void *stream);

/* Copy T_n from the device to the host copy (synchronises `stream`); optional T_out[batch]. */
int ripe_sync_lengths(ripe_cache_t *c, int32_t *T_out, void *stream);

/* Counters and geometry of the cache (host copy of the state; no device work). */
int ripe_cache_stats(const ripe_cache_t *c, ripe_stats *st);

/*
 * Logical view of one sequence of one layer, for tests: every position t < Tv = T_n + B
 * (B = block in flight, or 0) and every plane.
 *   k_out, v_out    device bf16 [R][kv_heads][Tv][d]; absent (position, plane) pairs are zero
 *   plane_present   device uint8 [R][Tv]; 1 where the cache stores that plane of that position
 * Requires synced lengths (RIPE_ESTATE otherwise).
 */
int ripe_cache_export(ripe_cache_t *c, int n, int layer, void *k_out, void *v_out,
                      uint8_t *plane_present, void *stream);

/* Read and clear the device error word (synchronises `stream`); *err_out gets its bits. */
int ripe_get_device_error(ripe_cache_t *c, uint32_t *err_out, void *stream);

/*
 * Allocation-free verification attention.  The paper has no counterpart: this entry point
 * exists for callers that cannot call cudaMalloc -- code whose device memory belongs to
 * someone else (an inference engine's memory pool, a framework that preallocates all device
 * memory) or code running while a stream capture is open, where allocation is not allowed.
 * It computes exactly what ripe_verify_attn computes, over cache buffers that the caller
 * owns and has filled in the documented layout, and allocates nothing.
 *
 * Its scratch (partial results of the split key ranges and their arrival counters) is one
 * file-scope device array of RIPE_STATIC_SCRATCH_BYTES, which every GPU that loads the
 * library holds until the process exits.  A problem whose scratch would exceed it is rejected
 * with RIPE_ESCRATCH: it needs (S + batch * kv_heads) * rows * (head_dim + 4) * 4 bytes plus
 * batch * kv_heads * 4, where S is the number of SMs and rows is 8, 16, 32 or 64 (the block
 * length times q_heads / kv_heads, rounded up to one of those).
 *
 * The first call on a device sets up that device (looks up the array's device address and
 * the SM count) with the device current; make that first call before any stream capture.
 * Every call shares the array and it keeps the last call's contents; each call tags the
 * counters with a call number of its own, so nothing is cleared in between (a call that passes
 * `device_error` enqueues only its kernel).  Calls that overlap on the GPU (other streams, or
 * other host threads) race on the array and must be serialised by the caller.
 * The view's buffers must stay valid until the work enqueued on `stream` has finished.
 * `device_error` (device uint32, optional) receives RIPE_DEVERR_* bits; the caller clears it.
 * Pass it: with NULL the bits go to a word inside the static array that the next call clears,
 * so a kernel that skipped its work (RIPE_DEVERR_CAPACITY: T + block_len > max_T for some
 * sequence; RIPE_DEVERR_WAIT_TIMEOUT) leaves out and lse unwritten without any trace.
 */
#define RIPE_STATIC_SCRATCH_BYTES (4u << 20)

typedef struct ripe_cache_view {
    int32_t batch, layers, q_heads, kv_heads, head_dim, loops; /* as for ripe_cache_alloc */
    int32_t window, max_T, max_B, window_mode;                  /* as for ripe_cache_alloc */
    int32_t block_len;       /* B of the block being verified (1 .. max_B) */
    const void *k_deep;      /* bf16 [layers][batch][kv_heads][max_T - W][head_dim], NULL when W >= max_T */
    const void *v_deep;
    const void *k_ring;      /* bf16 [layers][batch][loops][kv_heads][S][head_dim], S = min(W + max_B, max_T),
                                position t at slot t mod S */
    const void *v_ring;
    const int32_t *lengths;  /* device int32 [batch]: committed positions T_n */
} ripe_cache_view;

int ripe_verify_attn_static(const ripe_cache_view *view, int layer, int r, const void *q, void *out,
                            float *lse, float scale, uint32_t *device_error, void *stream);

/* How the library was built: RIPE_BUILD_* bits (no device work, no arguments). */
int ripe_build_info(void);

/* Which tensor-core consumer serves verification launches with 9..64 query rows per kv head
 * (launches with 1..8 rows, and those that write the draft block, always use mma.sync tiles). */
enum ripe_verify_consumer {
    RIPE_CONSUMER_DEFAULT = 0, /* mma.sync tiles: on B200 the faster one at every measured shape */
    RIPE_CONSUMER_MMA = 1,     /* mma.sync m16n8k16 tiles, accumulators in registers */
    RIPE_CONSUMER_TC = 2       /* tcgen05 MMAs with accumulators in tensor memory */
};
/* Process-wide choice for the launches enqueued after the call (every device, every cache and the
 * allocation-free entry point).  The initial value comes from the environment variable
 * RIPE_VERIFY_CONSUMER ("mma" or "tc"; unset or anything else: RIPE_CONSUMER_DEFAULT).
 * Returns the previous value, or RIPE_EINVAL (nothing changed) for a value outside the enum.
 * The two consumers agree within the bf16 output rounding, not bit for bit.  No device work. */
int ripe_set_verify_consumer(int consumer);
/* The current choice (RIPE_CONSUMER_*; no device work). */
int ripe_get_verify_consumer(void);

/* Number of kernel launches the library has enqueued since the cache was allocated. */
int64_t ripe_launch_count(const ripe_cache_t *c);

/* Static description of a status code. */
const char *ripe_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* RIPE_H */
