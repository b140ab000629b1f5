/*
 * moe.h -- C ABI of libmoe.so: a routed mixture-of-experts layer whose expert
 * weights live in pinned host memory and are cached, whole (layer, expert)
 * pair by pair, in a GPU-resident slot pool with one LRU policy shared by all
 * layers.  Single GPU (NVIDIA B200, sm_100a).
 *
 * What the layer computes, and where the FreeToken pages state it:
 *  - a router picks a few of many experts per token ("FreeToken linux",
 *    section "Como gestiona FreeToken la memoria MoE": 6 of 256 routed
 *    experts per layer for DeepSeek-V4-Flash);
 *  - the full expert set stays in host RAM, VRAM holds expert slots used as
 *    an LRU cache shared across MoE layers; a hit runs on the GPU, a miss is
 *    brought in over PCIe (same section and its memory-tier table;
 *    "FreeToken 290b model", section "Como gestiona FreeToken el prellenado
 *    y la decodificacion");
 *  - a cache entry is a logical (layer, expert) pair ("FreeToken rtx 4090",
 *    section "Como funciona la jerarquia de memoria MoE");
 *  - the cache can be resized at a scheduler safe point ("FreeToken
 *    quantization", section "Flujo de configuracion de la cuantizacion de
 *    FreeToken");
 *  - expert weights come as MXFP4, NVFP4 or BF16 ("FreeToken quantization",
 *    section "Formatos compatibles, hardware y perfil de rendimiento");
 *  - host expert banks are stored in the runtime's own layout so no
 *    repacking happens at start-up ("FreeToken linux", section "Prepara los
 *    pesos del modelo", the FTW format): moe_pack_expert produces that layout.
 * The pages print no formulas.  This library reads them as: softmax router
 * followed by top-k and renormalisation over the chosen k; SwiGLU experts
 * h = silu(W1 x) * (W3 x), y = W2 h; out = sum_j w_j y_j.
 *
 * Conventions for every entry point:
 *  - d_ marks a device pointer, h_ a host pointer.  The caller allocates and
 *    owns every buffer, device or host; the library never calls cudaMalloc,
 *    cudaFree or cudaHostAlloc.  It creates CUDA events for the cache.
 *  - `stream` arguments are cudaStream_t values passed as void*; NULL is the
 *    legacy default stream.
 *  - Work is enqueued asynchronously on the given stream unless stated.
 *  - Every function returns a moe_status; nothing aborts or prints.
 *    Argument errors are detected on the host before anything is enqueued.
 *  - Row-major everywhere.  Integer tensors are int32.  bf16 tensors are
 *    passed as uint16_t bit patterns.
 *  - Limits: hidden % 64 == 0, ffn % 64 == 0 (FP4 formats: hidden % 256 ==
 *    0 and ffn % 256 == 0), 1 <= top_k <= experts <= 4096, capacity <= 8192,
 *    layers * experts < 65536.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1,
    MOE_ERR_CAPACITY = -2,   /* a call requests more distinct experts than slots */
    MOE_ERR_CUDA = -3,       /* a CUDA runtime call or kernel launch failed */
    MOE_ERR_FILL = -4,       /* a miss fill could not be issued */
    MOE_ERR_TIMEOUT = -5,    /* reserved: a bounded device-side wait gave up */
    MOE_ERR_UNSUPPORTED = -6,/* shape or scale codes outside what the kernels handle */
    MOE_ERR_STATE = -7       /* the cache is in an unusable state */
} moe_status;

typedef enum { MOE_W_BF16 = 0, MOE_W_MXFP4 = 1, MOE_W_NVFP4 = 2 } moe_wfmt;
typedef enum { MOE_FILL_HOST = 0, MOE_FILL_DEVICE = 1 } moe_fill_mode;
typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1 } moe_dtype;

typedef struct {
    int32_t layers;   /* L: MoE layers sharing one cache */
    int32_t experts;  /* E: routed experts per layer */
    int32_t hidden;   /* H */
    int32_t ffn;      /* F: expert FFN width */
    int32_t top_k;    /* k */
    int32_t wfmt;     /* moe_wfmt */
} moe_shape;

typedef struct moe_cache moe_cache; /* opaque host-side handle */

/* Cache trace events, in the order one lookup emits them: every HIT in
 * ascending expert id, then for each miss in ascending expert id an EVICT
 * of its victim (if the slot was taken) followed by its MISS.  A resize
 * emits EVICT records for the surplus, then MOVE records for survivors
 * whose slot number changes. */
typedef enum { MOE_EV_HIT = 0, MOE_EV_MISS = 1, MOE_EV_EVICT = 2, MOE_EV_MOVE = 3 } moe_event;

typedef struct {
    uint32_t call;   /* LRU clock value of the call (1-based count of successful lookups) */
    int32_t slot;    /* slot the event refers to (for MOVE: the new slot) */
    uint16_t layer;  /* (layer, expert) key the event refers to */
    uint16_t expert;
    uint8_t event;   /* moe_event */
    uint8_t pad[3];
} moe_trace_rec;     /* 16 bytes */

typedef struct {
    uint64_t lookups;      /* successful lookup calls */
    uint64_t hits;         /* requested (layer, expert) pairs found resident */
    uint64_t misses;       /* requested pairs brought in */
    uint64_t evictions;
    uint64_t fill_bytes;   /* bytes copied host -> device by fills (both fill modes) */
    uint64_t host_syncs;   /* lookups that had to read the miss list on the host */
    uint64_t trace_dropped;/* records lost because the trace buffer was full */
} moe_cache_stats;

/* Profiling categories: kernels of each step, and the host->device fills. */
typedef enum {
    MOE_PROF_ROUTER = 0,  /* router logits + top-k kernels */
    MOE_PROF_LOOKUP = 1,  /* cache lookup kernel (or the decode front kernel), miss-group slot tables */
    MOE_PROF_PERMUTE = 2, /* histogram, scan, scatter/gather kernels */
    MOE_PROF_FFN = 3,     /* grouped FFN kernels (gate-up, down) */
    MOE_PROF_COMBINE = 4, /* combine kernel */
    MOE_PROF_FILL = 5,    /* miss fills: host->device copies, or the device-fill kernel */
    MOE_PROF_COUNT = 6
} moe_prof_kind;

typedef struct {
    uint64_t launches;  /* kernels launched (MOE_PROF_FILL: copies issued, or fill kernels) */
    uint64_t timed;     /* bracketed steps whose duration is in ms */
    double ms;          /* summed device time of the bracketed steps */
} moe_prof_entry;

/* Human-readable name of a status code (static string). */
const char* moe_status_str(int status);

/* Library version as major*10000 + minor*100 + patch. */
int moe_version(void);

/* ---------------------------------------------------------------- sizes */

/* Bytes of one packed expert blob (= one slot), a multiple of 128.
 * MXFP4, H=4096, F=2048: 13,369,344.  0 for an invalid shape. */
size_t moe_slot_bytes(const moe_shape* shape);

/* Device bytes the cache bookkeeping needs for `capacity` slots and a
 * trace buffer of `trace_capacity` records. */
size_t moe_cache_meta_bytes(const moe_shape* shape, int32_t capacity, int32_t trace_capacity);

/* Device workspace bytes of moe_permute for n tokens. */
size_t moe_permute_workspace_bytes(int32_t n, int32_t experts, int32_t top_k);

/* Device workspace bytes of moe_grouped_ffn for `rows` permuted rows. */
size_t moe_ffn_workspace_bytes(const moe_shape* shape, int32_t rows);

/* Device workspace bytes of moe_layer_forward for n tokens. */
size_t moe_layer_workspace_bytes(const moe_shape* shape, int32_t n);

/* Device workspace bytes of moe_prefill_forward for n tokens. */
size_t moe_prefill_workspace_bytes(const moe_shape* shape, int32_t n);

/* ---------------------------------------------------------------- packing */

/*
 * Host only.  Converts one expert from the canonical layout into the packed
 * slot blob (the device layout the kernels stream; its internal order is
 * private to this library and may change between versions).
 * Canonical layout:
 *   w13 [2F][H]: rows 0..F-1 gate W1, rows F..2F-1 up W3;  w2 [H][F].
 *   FP4 formats: two E2M1 codes per byte along a row, even column in the low
 *   nibble; w13_scales [2F][H/32] E8M0 (MXFP4) or [2F][H/16] E4M3 (NVFP4),
 *   w2_scales likewise over F.  NVFP4 also takes tensor_scales = {s13, s2}
 *   (fp32 scales of the whole W13 and W2); other formats ignore it (may be
 *   NULL).  BF16: w13/w2 are uint16 bit patterns, scales NULL.
 * blob_out: moe_slot_bytes(shape) bytes.
 * Errors: MOE_ERR_UNSUPPORTED for NaN scale codes (E8M0 255, E4M3
 * S.1111.111) or non-finite NVFP4 tensor scales.  Every other code is
 * accepted; a negative NVFP4 block scale is stored as its magnitude with the
 * block's 16 codes negated (exact).
 * Pages: the runtime keeps expert banks in its own layout so start-up does
 * no repacking ("FreeToken linux", section "Prepara los pesos del modelo",
 * the FTW format); the formats are named in "FreeToken quantization",
 * section "Formatos compatibles, hardware y perfil de rendimiento".
 */
int moe_pack_expert(const moe_shape* shape, const void* h_w13, const uint8_t* h_w13_scales,
                    const void* h_w2, const uint8_t* h_w2_scales, const float* h_tensor_scales,
                    void* h_blob_out);

/* ---------------------------------------------------------------- cache */

/*
 * Creates a cache of `capacity` slots over the caller's device memory
 * (pages: VRAM holds expert slots used as an LRU cache shared across MoE
 * layers while the full expert set stays in host RAM, "FreeToken linux",
 * section "Como gestiona FreeToken la memoria MoE"):
 *   d_meta: moe_cache_meta_bytes() bytes, 256-byte aligned;
 *   d_slot_pool: capacity * moe_slot_bytes() bytes, 256-byte aligned;
 *   h_blobs: layers*experts pointers, h_blobs[l*E+e] = packed blob of expert
 *   e of layer l in pinned host memory (the caller keeps the array and the
 *   blobs alive and unchanged for the life of the cache; several keys may
 *   point to the same blob).
 * All slots start free (cold cache).  Initialises d_meta on `stream` and
 * synchronises it.
 * Testing hook: with MOE_FAULT_INJECT=fill_fail:<n> in the environment when
 * the cache is created, the n-th fill (counting from 1, once) reports a failed
 * copy: the lookup that needed it returns MOE_ERR_FILL before any copy is
 * issued and its installs are rolled back.
 */
int moe_cache_create(const moe_shape* shape, void* d_meta, size_t meta_bytes, void* d_slot_pool,
                     int32_t capacity, int32_t trace_capacity, const void* const* h_blobs,
                     void* stream, moe_cache** out);

/*
 * Looks up the experts that `d_idx` (count entries, device, any order,
 * duplicates allowed) requests for `layer`, updates the LRU state (the
 * policy is stated on moe_trace_rec and below), records the trace, and
 * brings every miss into its slot.
 *   LRU: the clock advances by one per successful call; hits get the new
 *   clock value; each miss (ascending expert id) takes the lowest free slot,
 *   else evicts the resident key with the smallest (last use, slot) that
 *   this call does not request.
 * d_slot_of_expert [E] (device) receives the slot of each requested expert,
 * -1 for the others.  Fills are issued on copy_stream after everything
 * already on `stream` is done, and `stream` waits for them, so work enqueued
 * on `stream` afterwards sees the weights.
 * Host fills (the default): blocks the host until the miss list is known,
 * except when every expert of `layer` is already resident (then nothing is
 * read back).  MOE_ERR_CAPACITY if more distinct experts are requested than
 * slots exist; the state is unchanged (the host learns this at the same sync
 * point).  Device fills (moe_cache_set_fill_mode): never blocks; the fill
 * kernel runs on copy_stream and `stream` waits for it; a capacity error
 * leaves the state unchanged, every slot_of entry -1, and is reported by
 * moe_cache_device_status.
 * Pages: hits run directly on the GPU and misses are brought in ("FreeToken
 * 290b model", section "Como gestiona FreeToken el prellenado y la
 * decodificacion"); a cache entry is a logical (layer, expert) pair
 * ("FreeToken rtx 4090", section "Como funciona la jerarquia de memoria
 * MoE").
 */
int moe_cache_lookup_update(moe_cache* cache, int32_t layer, const int32_t* d_idx, int32_t count,
                            int32_t* d_slot_of_expert, void* stream, void* copy_stream);

/*
 * Resizes the cache to new_capacity slots at a safe point: synchronises
 * `stream`, evicts the least recently used surplus (by (last use, slot)),
 * copies the survivors, packed to the front in old-slot order, into
 * d_pool_new, and moves the bookkeeping to d_meta_new (either may equal the
 * old buffer when large enough; the survivors only ever move to lower
 * slots, so an in-place pool works).  Emits EVICT / MOVE trace records.
 * Pages: the cache is rebuilt at scheduler safe points ("FreeToken
 * quantization", section "Flujo de configuracion de la cuantizacion de
 * FreeToken").
 */
int moe_cache_resize(moe_cache* cache, void* d_meta_new, size_t meta_bytes, void* d_pool_new,
                     int32_t new_capacity, void* stream);

/*
 * Chooses how misses are brought in (default MOE_FILL_HOST).
 *   MOE_FILL_HOST: the host reads the lookup's miss list back and issues one
 *   cudaMemcpyAsync per miss on copy_stream (the DMA engine).
 *   MOE_FILL_DEVICE: a copy kernel on copy_stream reads the miss list where
 *   the lookup kernel wrote it and copies each missing blob from pinned host
 *   memory, mapped into the device's address space, into its slot (zero-copy
 *   loads over PCIe by 16 CTAs; moe_layer_forward launches it once per miss
 *   group, each launch copying its group's part of the list).  No call reads
 *   anything back, so
 *   moe_cache_lookup_update and moe_layer_forward never block the host and a
 *   whole decode step, misses included, can be captured in a CUDA graph.
 *   The kernel waits for nothing on the device (stream order sequences it
 *   after the lookup and before the misses' FFN passes), so it has no timeout.
 *   Requires every blob of h_blobs to be 16-byte aligned page-locked host
 *   memory mapped into the device's address space (cudaHostAlloc /
 *   cudaMallocHost memory on a system with unified addressing, or
 *   cudaHostRegister with cudaHostRegisterMapped), the whole blob inside one
 *   mapping; otherwise MOE_ERR_INVALID_ARG and the mode is unchanged.  The
 *   fill_fail testing hook of moe_cache_create applies to host fills only.
 * The trace, the LRU state and the results are the same in both modes.
 * Synchronises `stream`; call it at a safe point (no call of this cache in
 * flight).
 * Pages: misses are brought over PCIe from the host expert set into VRAM
 * ("FreeToken 290b model", section "Como gestiona FreeToken el prellenado y
 * la decodificacion"); who issues the copy is this library's choice.
 */
int moe_cache_set_fill_mode(moe_cache* cache, int32_t mode, void* stream);

/* The current moe_fill_mode, or MOE_ERR_INVALID_ARG for a NULL cache. */
int32_t moe_cache_fill_mode(const moe_cache* cache);

/* First error a lookup kernel recorded since the last clear (MOE_ERR_CAPACITY,
 * or MOE_ERR_INVALID_ARG for an expert index outside [0, E)), 0 if none;
 * clear != 0 resets it.  The way to learn of a failed lookup under device
 * fills, where calls do not read the lookup's status back.  Synchronous. */
int moe_cache_device_status(moe_cache* cache, int32_t clear);

/* Copies up to `cap` trace records, oldest first, into h_buf, reports how
 * many in *n_out, and clears the device trace buffer.  Synchronous. */
int moe_cache_read_trace(moe_cache* cache, moe_trace_rec* h_buf, size_t cap, size_t* n_out);

/* Counters since creation.  Synchronous. */
int moe_cache_get_stats(moe_cache* cache, moe_cache_stats* out);

/* Host copies of the slot table [L*E], slot keys [C] (l*E+e or -1) and
 * last-use stamps [C].  Any pointer may be NULL.  Synchronous. */
int moe_cache_snapshot(moe_cache* cache, int32_t* h_slot_of, int32_t* h_key_of, uint64_t* h_stamp);

int32_t moe_cache_capacity(const moe_cache* cache);

/* Releases the host-side handle and its events (not the caller's memory). */
int moe_cache_destroy(moe_cache* cache);

/* ---------------------------------------------------------------- steps */

/*
 * Router.  d_x [n][hidden] (float32 or bf16 per x_dtype), d_wg [experts]
 * [hidden] bf16, d_bias [experts] float32 or NULL.
 *   logit[t][e] = fp32(sum_h x[t][h] * wg[e][h]) + bias[e], the sum formed in
 *   a fixed order: 32 lanes, lane l accumulating with fused multiply-adds
 *   over the 8-element chunks l, l+32, ... in ascending order, then an xor
 *   butterfly (16, 8, 4, 2, 1) across the lanes.
 *   d_topk_idx [n][k]: the k largest logits, descending; ties go to the
 *   lower expert id; NaN ranks below -inf.
 *   d_topk_w [n][k]: exp(l_j - l_max) / sum over the chosen k (softmax over
 *   all experts renormalised over the top-k).
 * d_logits [n][experts] float32 is scratch the caller provides, and holds
 * the logits afterwards.
 * Pages: each token is sent to a few of a layer's routed experts (6 of 256
 * for DeepSeek-V4-Flash, "FreeToken linux", section "Como gestiona
 * FreeToken la memoria MoE"); the softmax / top-k / renormalisation reading
 * is this library's (the pages print no formula).
 */
int moe_router_topk(const void* d_x, int32_t x_dtype, const uint16_t* d_wg, const float* d_bias,
                    int32_t n, int32_t hidden, int32_t experts, int32_t k, float* d_logits,
                    int32_t* d_topk_idx, float* d_topk_w, void* stream);

/*
 * Token -> expert permutation.  Assignment a = t*k + j goes to expert
 * idx[a].  d_expert_offsets [experts+1]: exclusive prefix sum of the
 * per-expert counts; d_row_of [n*k]: row_of[a] = offsets[e] + number of
 * earlier assignments to the same expert (stable); d_assign_of [n*k]: the
 * inverse; d_x_perm [n*k][hidden] bf16: x_perm[row_of[a]] = bf16(x[a/k])
 * (round to nearest even when x is float32).  d_ws: workspace of
 * moe_permute_workspace_bytes() bytes.  An index outside [0, experts) is
 * the caller's error: that assignment gets row_of = -1 and no row, and
 * offsets[experts] counts only the valid ones.
 * Pages: no passage; the step that groups each expert's tokens so the
 * experts run as a grouped GEMM.
 */
int moe_permute(const int32_t* d_topk_idx, int32_t n, int32_t experts, int32_t k, const void* d_x,
                int32_t x_dtype, int32_t hidden, int32_t* d_expert_offsets, int32_t* d_row_of,
                int32_t* d_assign_of, uint16_t* d_x_perm, void* d_ws, size_t ws_bytes,
                void* stream);

/*
 * moe_permute without a caller-provided workspace.  No counterpart on the
 * FreeToken pages: this is a convenience for callers that cannot allocate
 * device memory of their own -- for example code running inside a host
 * framework whose allocator owns all GPU memory and forbids foreign
 * cudaMalloc calls, or a latency-critical serving loop that must never enter
 * the CUDA allocator (cudaMalloc / cudaFree may synchronise the device).
 * Arguments, outputs and ordering are those of moe_permute.
 * The scratch is one static device array of MOE_PERMUTE_NOALLOC_MAX_SCRATCH
 * bytes inside libmoe.so, present on every GPU that loads the library for the
 * life of the process.  The first call on a device looks the array's device
 * address up (with that device current); make that first call before any
 * stream capture.  Allocates nothing: no cudaMalloc, cudaFree or other
 * allocating routine.  Nothing in the array has to start at zero: every
 * entry a call reads is written earlier in that same call, so leftovers of a
 * previous call are harmless.  Sizes whose moe_permute_workspace_bytes() exceed the
 * array return MOE_ERR_UNSUPPORTED before anything is enqueued.  All calls on
 * a device share the one array: calls that may overlap on the GPU (different
 * streams, or other host threads) race and must be serialised by the caller.
 */
#define MOE_PERMUTE_NOALLOC_MAX_SCRATCH (1u << 20)
int moe_permute_noalloc(const int32_t* d_topk_idx, int32_t n, int32_t experts, int32_t k, const void* d_x,
                        int32_t x_dtype, int32_t hidden, int32_t* d_expert_offsets, int32_t* d_row_of,
                        int32_t* d_assign_of, uint16_t* d_x_perm, void* stream);

/*
 * Grouped SwiGLU expert FFN over the permuted rows.  d_slot_pool holds
 * pool_slots packed blobs of moe_slot_bytes() each.  d_expert_offsets holds
 * E+1 non-decreasing values with offsets[0] >= 0 and offsets[E] <= rows (the
 * exclusive prefix sums moe_permute writes); other contents are undefined
 * behaviour.  For every expert e with rows [offsets[e], offsets[e+1]) and
 * 0 <= d_slot_of_expert[e] < pool_slots, the weights are read from that
 * slot and
 *   h = silu(x W1^T) * (x W3^T)   (fp32 accumulation),
 *   y = h W2^T                    (fp32 accumulation, y rounded to bf16)
 * is written to d_y_perm rows.  Rows of experts with any other slot value
 * (-1 in particular), or whose range does not lie inside [0, rows), are left
 * untouched, so hits and misses can run as two passes.
 * d_ws: moe_ffn_workspace_bytes() bytes.
 * FP4 weights (MXFP4, NVFP4) run on the block-scaled tensor cores: the E2M1
 * weights and their block scales are multiplied as stored; each x and h row
 * is first written as T E2M1 terms with block scales of the weights' scale
 * type (moe_act_terms: T = 4 when the call has few rows per expert, 3 when
 * it averages at least 4; relative error about 2e-4 and 2e-3 per row), the
 * terms' products are summed in fp32, and the NVFP4 row and tensor scales
 * are undone in fp32.  BF16 weights run on bf16 MMAs with x and h rounded to
 * bf16.  Results are deterministic: the same inputs give the same bits on
 * every call.  MOE_FFN_TILE=decode or =prefill forces the FP4 tile shape
 * (read at every call; intended for testing).  FP4 calls with decode tiles
 * run as one cooperative kernel whose grid barriers use a process-wide
 * counter of the device: such calls must not run at the same time on
 * different streams (calls on one stream never do).
 * Pages: experts found in VRAM execute on the GPU ("FreeToken
 * quantization", section "Como se desplazan los pesos MoE cuantizados por la
 * memoria"); SwiGLU is this library's reading (the pages name no
 * activation).
 */
int moe_grouped_ffn(const moe_shape* shape, const void* d_slot_pool, int32_t pool_slots,
                    const int32_t* d_slot_of_expert, const int32_t* d_expert_offsets,
                    const uint16_t* d_x_perm, int32_t rows, uint16_t* d_y_perm, void* d_ws,
                    size_t ws_bytes, void* stream);

/*
 * Combine.  out[t] = sum over j = 0..k-1, in that order, of
 * w[t][j] * y_perm[row_of[t*k+j]], accumulated in fp32 and stored as
 * out_dtype.  Deterministic (no atomics).
 * Pages: no passage; the gate-weighted sum of a routed MoE layer.
 */
int moe_combine(const uint16_t* d_y_perm, const int32_t* d_row_of, const float* d_topk_w, int32_t n,
                int32_t k, int32_t hidden, void* d_out, int32_t out_dtype, void* stream);

/*
 * The whole layer for `layer`: router -> cache lookup -> permute -> grouped
 * FFN over the hits -> (fills of the misses on copy_stream, overlapped with
 * the hit FFN) -> grouped FFN over the misses -> combine.
 * Misses run in up to 4 miss groups in miss-list order (the last groups one
 * miss each; with nm misses the first non-empty group holds nm - 3 when
 * nm > 4): each group's FFN call starts once its own blobs have landed, so
 * only the last miss's FFN follows the last fill.  Results depend on the
 * grouping (the FFN's split of the work over the SMs does), and are the same
 * in both fill modes.
 * d_x [n][H] (x_dtype), d_wg [E][H] bf16, d_bias [E] or NULL; d_out [n][H]
 * in x_dtype.  d_ws: moe_layer_workspace_bytes() bytes.  d_topk_idx_out /
 * d_topk_w_out ([n][k], device) receive the routing when not NULL.
 * Calls of at most 32 tokens (with E <= 1024 and n*k <= 1024) run the top-k,
 * the lookup and the permutation as one kernel after the logits kernel; the
 * results are those of the separate steps.
 * Host fills: blocks the host once, for the miss list, unless every expert
 * of the layer is resident; in that case nothing is read back and the call
 * can be captured in a CUDA graph.  Device fills (moe_cache_set_fill_mode):
 * the fill kernel runs on copy_stream beside the hit FFN, nothing is read
 * back, and every call can be captured in a CUDA graph.
 * Pages: hits execute on the GPU while misses are brought in ("FreeToken
 * 290b model", section "Como gestiona FreeToken el prellenado y la
 * decodificacion"); data movement overlaps computation ("FreeToken linux",
 * mechanism table in section "Como gestiona FreeToken la memoria MoE").
 */
int moe_layer_forward(moe_cache* cache, int32_t layer, const void* d_x, int32_t x_dtype,
                      const uint16_t* d_wg, const float* d_bias, int32_t n, void* d_out,
                      void* d_ws, size_t ws_bytes, void* stream, void* copy_stream,
                      int32_t* d_topk_idx_out, float* d_topk_w_out);

/*
 * Multi-layer prefill with full-layer double buffering: layers layer0 ..
 * layer0 + n_layers - 1 over one prompt of n tokens, every expert of a layer
 * brought into the cache before the layer runs.  Layer i of the call (layer
 * l = layer0 + i) reads d_x[i] [n][H] (x_dtype), its router d_wg[i] [E][H]
 * bf16 and d_bias[i] [E] (d_bias, or any entry, may be NULL), and writes
 * d_out[i] [n][H] (x_dtype) and, when d_topk_idx_out is not NULL, its
 * routing to d_topk_idx_out + i*n*k.  d_x, d_wg, d_bias and d_out are host
 * arrays of n_layers device pointers; d_x[i+1] may be d_out[i].  Each layer
 * computes what moe_layer_forward computes.
 * Cache: one lookup per layer, in layer order, requesting all E experts
 * (ascending), with the LRU updates, trace records and fills of
 * moe_cache_lookup_update in the cache's fill mode.  With capacity >= 2E the
 * lookup and fills of layer l+1 are issued before layer l computes, so the
 * next layer's experts stream over PCIe on copy_stream while the current one
 * computes; the LRU order keeps layer l's slots out of their victims (layer
 * l's keys are the newest, and at least E slots are free or older).  With
 * E <= capacity < 2E the next layer's lookup follows the current layer's
 * compute (no overlap).  MOE_ERR_CAPACITY (before anything is enqueued) when
 * capacity < E.  Host fills block the host at every lookup that may miss,
 * until the previous layer's fills have landed; device fills never block.
 * d_ws: moe_prefill_workspace_bytes(shape, n) bytes.  Pointers 16-byte
 * aligned.
 * Pages: during prefill the whole next layer's experts stream over PCIe into
 * a second buffer while the GPU computes the current layer, when the cache
 * has room for it ("FreeToken linux", section "Como gestiona FreeToken la
 * memoria MoE" and its mechanism table, "Doble bufer para la capa
 * completa"; "FreeToken 290b model", section "Como gestiona FreeToken el
 * prellenado y la decodificacion"); the same cache serves prefill and decode
 * (same section of "FreeToken linux").
 */
int moe_prefill_forward(moe_cache* cache, int32_t layer0, int32_t n_layers, const void* const* d_x,
                        int32_t x_dtype, const uint16_t* const* d_wg, const float* const* d_bias, int32_t n,
                        void* const* d_out, void* d_ws, size_t ws_bytes, void* stream, void* copy_stream,
                        int32_t* d_topk_idx_out);

/*
 * The operand encoding the FP4 grouped FFN applies to its activation rows,
 * exposed for inspection and testing: d_x [rows][K] (x_dtype, K % 32 == 0,
 * 16-byte aligned).  For wfmt MXFP4 every 32-column block, for NVFP4 every
 * 16-column block, is written as `terms` (3 or 4) E2M1 terms, each with its
 * own block scale (E8M0, resp. unsigned E4M3): term t takes the smallest
 * scale s of the format with 6 s >= the block's largest remaining
 * magnitude m (E8M0 codes 1..254; E4M3 codes 1..0x7E against m / 6 in
 * fp32; code 127 / 0x38 when m is 0), the E2M1 code nearest to r / s (ties
 * to the even code) for each element, and leaves r - e2m1 * s to the next
 * term, all in fp32.  NVFP4 rows are first multiplied by 2^p with 2^p times
 * the row's largest magnitude in [2^10, 2^11) (p clamped to [-100, 100]).
 * Outputs (device): d_codes [rows][terms][K] one code per byte,
 * d_scales [rows][terms][K / vs] scale codes, d_row_exp [rows] p (0 for
 * MXFP4).  Row i is 2^-p sum_t e2m1(codes) * scale.  Errors:
 * MOE_ERR_INVALID_ARG for bad sizes, dtypes or pointers, MOE_ERR_UNSUPPORTED
 * for other term counts.
 * Pages: none; the pages name the weight formats ("FreeToken quantization",
 * section "Formatos compatibles, hardware y perfil de rendimiento"), this
 * encoding is how this library feeds them to FP4 tensor cores.
 */
int moe_act_terms(const void* d_x, int32_t x_dtype, int32_t rows, int32_t K, int32_t wfmt, int32_t terms,
                  uint8_t* d_codes, uint8_t* d_scales, int32_t* d_row_exp, void* stream);

/* ---------------------------------------------------------------- profiling */

/*
 * Launch counters are always kept (process-wide).  With timing != 0, every
 * step an entry point enqueues (the router's two kernels, the lookup, the
 * permutation's three kernels, each grouped-FFN pass, the combine, each
 * call's batch of fills) is bracketed by two CUDA events recorded on the
 * stream it runs on.  Not thread-safe with respect to moe_profile_read.
 */
int moe_profile_enable(int timing);

/* Waits for the pending events, then copies min(count, MOE_PROF_COUNT)
 * entries (indexed by moe_prof_kind) to h_out; reset != 0 zeroes all
 * counters afterwards.  Synchronous. */
int moe_profile_read(moe_prof_entry* h_out, int count, int reset);

/*
 * First error recorded by a device-side bounded wait since the last clear
 * (MOE_ERR_TIMEOUT when a kernel gave up waiting and drained instead of
 * hanging), 0 if none; clear != 0 resets it.  Synchronous.  The grouped FFN
 * results of a call that timed out, and of FP4 decode calls made while the
 * error is set (their grid barriers give up at once), are undefined; clear
 * the error before relying on results again.
 */
int moe_get_device_error(int clear);

/*
 * Testing hook, process-wide, for grouped-FFN launches made afterwards:
 * `cycles` > 0 sets the limit of the kernels' bounded waits to that many SM
 * clock cycles (0 restores the default of about 2 s), and withhold != 0
 * makes the first CTA's copy issuer leave its first ring stage unfilled, so
 * that the wait for it runs out: the kernel records MOE_ERR_TIMEOUT, lets
 * its own copies and MMAs finish and returns.  Drains of a CTA's own
 * asynchronous work keep the default limit.  MOE_ERR_INVALID_ARG for
 * cycles < 0.  Not thread-safe with concurrent launches.
 * Pages: none (a robustness test of this library's bounded waits).
 */
int moe_test_set_wait(int64_t cycles, int32_t withhold);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
