// The whole routed MoE layer chained on one compute stream, with miss fills
// on a copy stream overlapped with the FFN over the hits.
//
// Pages: during decode the routed experts are checked in the GPU cache, hits
// execute directly on the GPU and misses are brought in ("FreeToken 290b
// model", section "Como gestiona FreeToken el prellenado y la
// decodificacion"); data movement is overlapped with computation instead of
// leaving the GPU idle ("FreeToken linux", mechanism table in section "Como
// gestiona FreeToken la memoria MoE").  Splitting misses between fills and
// CPU execution is not done here: every miss is filled and runs on the GPU.
#include "common.cuh"

namespace moe {
struct LayerWs {
    float* logits;
    int32_t* idx;
    float* w;
    int32_t* offsets;
    int32_t* row_of;
    int32_t* assign_of;
    uint16_t* y_perm;
    int32_t* grp_slots;   // [kMissGroups][E]: slot tables of the miss groups
    void* ffn_ws;
    void* perm_ws;
    size_t bytes;
};

static LayerWs layer_ws(const moe_shape* s, int n, void* base)
{
    LayerWs L{};
    const size_t A = (size_t)n * s->top_k, E = s->experts, H = s->hidden;
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align_up(o + b, 256); return at; };
    size_t o_logits = take(4 * (size_t)n * E);
    size_t o_idx = take(4 * A);
    size_t o_w = take(4 * A);
    size_t o_off = take(4 * (E + 1));
    size_t o_row = take(4 * A);
    size_t o_asg = take(4 * A);
    size_t o_yp = take(2 * A * H);
    size_t o_grp = take(4 * (size_t)kMissGroups * E);
    size_t o_ffn = take(ffn_ws_bytes(s, (int)A));
    size_t o_perm = take(permute_ws_bytes(n, s->experts, s->top_k));
    L.bytes = o;
    if (base) {
        char* b = static_cast<char*>(base);
        L.logits = reinterpret_cast<float*>(b + o_logits);
        L.idx = reinterpret_cast<int32_t*>(b + o_idx);
        L.w = reinterpret_cast<float*>(b + o_w);
        L.offsets = reinterpret_cast<int32_t*>(b + o_off);
        L.row_of = reinterpret_cast<int32_t*>(b + o_row);
        L.assign_of = reinterpret_cast<int32_t*>(b + o_asg);
        L.y_perm = reinterpret_cast<uint16_t*>(b + o_yp);
        L.grp_slots = reinterpret_cast<int32_t*>(b + o_grp);
        L.ffn_ws = b + o_ffn;
        L.perm_ws = b + o_perm;
    }
    return L;
}

// Router -> permutation -> grouped FFN over the experts in `slot_of` ->
// combine, for one layer whose experts are already in their slots.
static int layer_chain(const moe_shape* s, const LayerWs& L, const char* pool, size_t sb, int C,
                       const int32_t* slot_of, const void* x, int x_dtype, const uint16_t* wg, const float* bias,
                       int n, void* out, int32_t* idx, float* w, cudaStream_t st)
{
    const int E = s->experts, k = s->top_k, H = s->hidden, A = n * k;
    int rc;
    if ((rc = launch_router(x, x_dtype, wg, bias, n, H, E, k, L.logits, idx, w, st))) return rc;
    if ((rc = launch_permute(idx, n, E, k, x, x_dtype, H, L.offsets, L.row_of, L.assign_of, nullptr, L.perm_ws, st)))
        return rc;
    const RowSource src{x, x_dtype, L.assign_of, k};
    if ((rc = launch_ffn(s, pool, sb, C, slot_of, L.offsets, nullptr, A, L.y_perm, L.ffn_ws, st, &src))) return rc;
    return launch_combine(L.y_perm, L.row_of, w, n, k, H, out, x_dtype, st);
}

// Prefill workspace: one layer's, then the expert list 0..E-1 and the slot
// tables of the two layers in flight.
struct PrefillWs {
    LayerWs L;
    int32_t* all;
    int32_t* slot[2];
    size_t bytes;
};

static PrefillWs prefill_ws(const moe_shape* s, int n, void* base)
{
    PrefillWs P{};
    P.L = layer_ws(s, n, base);
    const size_t e4 = align_up(4 * (size_t)s->experts, 256);
    P.bytes = P.L.bytes + 3 * e4;
    if (base) {
        char* b = static_cast<char*>(base) + P.L.bytes;
        P.all = reinterpret_cast<int32_t*>(b);
        P.slot[0] = reinterpret_cast<int32_t*>(b + e4);
        P.slot[1] = reinterpret_cast<int32_t*>(b + 2 * e4);
    }
    return P;
}

__global__ void iota_kernel(int32_t* v, int n)
{
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) v[i] = i;
}

}  // namespace moe

using namespace moe;

extern "C" size_t moe_prefill_workspace_bytes(const moe_shape* shape, int32_t n)
{
    if (!shape_ok(shape) || n < 0) return 0;
    return prefill_ws(shape, n, nullptr).bytes;
}

extern "C" int moe_prefill_forward(moe_cache* c, int32_t layer0, int32_t n_layers, const void* const* d_x,
                                   int32_t x_dtype, const uint16_t* const* d_wg, const float* const* d_bias,
                                   int32_t n, void* const* d_out, void* d_ws, size_t ws_bytes, void* stream,
                                   void* copy_stream, int32_t* d_topk_idx_out)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    const moe_shape* s = cache_shape(c);
    if (layer0 < 0 || n_layers < 0 || layer0 + (int64_t)n_layers > s->layers || n < 0) return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n_layers == 0 || n == 0) return MOE_OK;
    if (!d_x || !d_wg || !d_out || !d_ws) return MOE_ERR_INVALID_ARG;
    for (int i = 0; i < n_layers; i++) {
        if (!d_x[i] || !d_wg[i] || !d_out[i]) return MOE_ERR_INVALID_ARG;
        if (((uintptr_t)d_x[i] | (uintptr_t)d_wg[i] | (uintptr_t)d_out[i]) & 15) return MOE_ERR_INVALID_ARG;
    }
    if ((uintptr_t)d_ws & 15) return MOE_ERR_INVALID_ARG;
    const PrefillWs P = prefill_ws(s, n, d_ws);
    if (ws_bytes < P.bytes) return MOE_ERR_INVALID_ARG;
    const int E = s->experts, k = s->top_k, C = cache_capacity_int(c);
    if (C < E) return MOE_ERR_CAPACITY;   // a whole layer must fit
    // Two whole layers fit: the next layer's lookup goes ahead of this
    // layer's compute.  Its misses take the least recently used slots that
    // it does not request; this layer's keys carry the newest stamps and at
    // least E older keys or free slots exist, so none of them is a victim.
    const bool overlap = C >= 2 * E;
    cudaStream_t st = as_stream(stream), cp = as_stream(copy_stream);
    const char* pool = cache_pool(c);
    const size_t sb = cache_slot_bytes(c);
    int rc;
    iota_kernel<<<(E + 255) / 256, 256, 0, st>>>(P.all, E);
    MOE_LAUNCH_CHECK();
    auto bring_in = [&](int l, int b) -> int {
        int r = cache_launch_lookup(c, l, P.all, E, P.slot[b], st);
        return r ? r : cache_fill(c, l, st, cp, cache_prefill_event(c, b));
    };
    if ((rc = bring_in(layer0, 0))) return rc;
    for (int i = 0; i < n_layers; i++) {
        const int l = layer0 + i, b = i & 1;
        // this layer's fills have landed (and device fills have read the
        // miss list, which the next lookup rewrites) before anything else
        // on the compute stream; the compute needs them anyway
        MOE_CUDA_TRY(cudaStreamWaitEvent(st, cache_prefill_event(c, b), 0));
        if (overlap && i + 1 < n_layers && (rc = bring_in(l + 1, b ^ 1))) return rc;
        int32_t* idx = d_topk_idx_out ? d_topk_idx_out + (size_t)i * n * k : P.L.idx;
        if ((rc = layer_chain(s, P.L, pool, sb, C, P.slot[b], d_x[i], x_dtype, d_wg[i], d_bias ? d_bias[i] : nullptr,
                              n, d_out[i], idx, P.L.w, st)))
            return rc;
        if (!overlap && i + 1 < n_layers && (rc = bring_in(l + 1, b ^ 1))) return rc;
    }
    return MOE_OK;
}

extern "C" size_t moe_layer_workspace_bytes(const moe_shape* shape, int32_t n)
{
    if (!shape_ok(shape) || n < 0) return 0;
    return layer_ws(shape, n, nullptr).bytes;
}

extern "C" int moe_layer_forward(moe_cache* c, int32_t layer, const void* d_x, int32_t x_dtype, const uint16_t* d_wg,
                                 const float* d_bias, int32_t n, void* d_out, void* d_ws, size_t ws_bytes,
                                 void* stream, void* copy_stream, int32_t* d_topk_idx_out, float* d_topk_w_out)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    const moe_shape* s = cache_shape(c);
    if (layer < 0 || layer >= s->layers || n < 0) return MOE_ERR_INVALID_ARG;
    if (x_dtype != MOE_DT_F32 && x_dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
    if (n > 0 && (!d_x || !d_wg || !d_out || !d_ws)) return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_x | (uintptr_t)d_wg | (uintptr_t)d_out | (uintptr_t)d_ws) & 15) return MOE_ERR_INVALID_ARG;
    LayerWs L = layer_ws(s, n, d_ws);
    if (ws_bytes < L.bytes) return MOE_ERR_INVALID_ARG;
    if (n == 0) return MOE_OK;
    cudaStream_t st = as_stream(stream), cp = as_stream(copy_stream);
    const int E = s->experts, k = s->top_k, H = s->hidden, A = n * k;
    int32_t* idx = d_topk_idx_out ? d_topk_idx_out : L.idx;
    float* w = d_topk_w_out ? d_topk_w_out : L.w;
    int rc;
    // Both FFN paths gather the token rows straight from x into their own
    // operand copies, so the permutation writes no x_perm.
    uint16_t* xp = nullptr;
    if (cache_front_fits(c, n)) {
        // decode-sized calls: top-k, lookup and permutation in one launch after the logits
        if ((rc = launch_router_logits(d_x, x_dtype, d_wg, d_bias, n, H, E, L.logits, st))) return rc;
        if ((rc = cache_launch_front(c, layer, L.logits, n, idx, w, L.offsets, L.row_of, L.assign_of, st)))
            return rc;
    } else {
        if ((rc = launch_router(d_x, x_dtype, d_wg, d_bias, n, H, E, k, L.logits, idx, w, st))) return rc;
        if ((rc = cache_launch_lookup(c, layer, idx, A, nullptr, st))) return rc;
        if ((rc = launch_permute(idx, n, E, k, d_x, x_dtype, H, L.offsets, L.row_of, L.assign_of, xp, L.perm_ws, st)))
            return rc;
    }
    const RowSource src{d_x, x_dtype, L.assign_of, k};
    const RowSource* gather = &src;
    const char* pool = cache_pool(c);
    const size_t sb = cache_slot_bytes(c);
    const int C = cache_capacity_int(c);
    const bool dev_fill = cache_fill_mode(c) == MOE_FILL_DEVICE;
    if (!dev_fill && cache_layer_resident(c, layer)) {
        // every expert of this layer is resident: no miss is possible, nothing is read back
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_all(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
    } else {
        // Device fills take the miss list from the lookup on the device: the
        // copy kernels start first (few SMs, only PCIe) and nothing is read
        // back.  Host fills: the hits run while the host learns the miss list
        // and issues the copies.  Either way the misses run in miss groups,
        // each as soon as its blobs have landed, so the FFN of all but the
        // last miss overlaps the later copies.
        unsigned live = 0;
        if (dev_fill && (rc = cache_group_fills(c, layer, st, cp, &live))) return rc;
        if ((rc = launch_ffn(s, pool, sb, C, cache_slot_hit(c), L.offsets, xp, A, L.y_perm, L.ffn_ws, st, gather)))
            return rc;
        if (!dev_fill && (rc = cache_group_fills(c, layer, st, cp, &live))) return rc;
        if (live) {
            if ((rc = cache_launch_group_slots(c, L.grp_slots, st))) return rc;
            for (int g = 0; g < kMissGroups; g++) {
                if (!((live >> g) & 1)) continue;
                MOE_CUDA_TRY(cudaStreamWaitEvent(st, cache_group_event(c, g), 0));
                // groups after the first hold one miss at most (miss_group)
                if ((rc = launch_ffn(s, pool, sb, C, L.grp_slots + (size_t)g * E, L.offsets, xp, A, L.y_perm,
                                     L.ffn_ws, st, gather, g > 0)))
                    return rc;
            }
        }
    }
    return launch_combine(L.y_perm, L.row_of, w, n, k, H, d_out, x_dtype, st);
}

extern "C" const char* moe_status_str(int status)
{
    switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_CAPACITY: return "more distinct experts requested than cache slots";
    case MOE_ERR_CUDA: return "CUDA runtime error";
    case MOE_ERR_FILL: return "expert fill failed";
    case MOE_ERR_TIMEOUT: return "device wait timed out";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or scale codes";
    case MOE_ERR_STATE: return "cache state error";
    }
    return "unknown status";
}

extern "C" int moe_version(void) { return 100; }
