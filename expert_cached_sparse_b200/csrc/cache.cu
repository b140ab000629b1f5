// GPU-resident expert-slot cache: one LRU over (layer, expert) keys shared
// by all MoE layers, misses filled from pinned host memory by async copies.
//
// Pages: the full expert set stays in system memory and VRAM is used as an
// elastic cache with an LRU policy shared across MoE layers; a hit runs on
// the GPU, a miss is brought over PCIe ("FreeToken linux", section "Como
// gestiona FreeToken la memoria MoE", and its memory-tier table).  A cache
// entry is one logical (layer, expert) pair ("FreeToken rtx 4090", section
// "Como funciona la jerarquia de memoria MoE").  Pinned host memory for DMA
// ("FreeToken 290b model", section "Prepara el conjunto de expertos del
// host").  Resize at scheduler safe points ("FreeToken quantization",
// section "Flujo de configuracion de la cuantizacion de FreeToken").
//
// Two ways to bring misses in.  Host fills: the host reads the miss list
// back and issues one DMA copy per miss.  Device fills: a copy kernel reads
// the miss list where the lookup kernel left it and loads each blob from
// pinned host memory mapped into the device's address space (zero-copy
// loads over PCIe), so no call blocks and a decode step with misses can be
// captured in a CUDA graph.
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "common.cuh"
#include "route_dev.cuh"

namespace moe {

// -------------------------------------------------------------- device meta layout
struct LookupHdr {          // written by every lookup, read back by the host
    int32_t status;
    uint32_t clock;
    int32_t n_req, n_hit, n_miss, n_evict;
    int32_t n_free;         // free slots before the call
    int32_t sticky;         // first device-side error seen (0 if none)
};
struct MissEnt {
    int32_t expert, slot, old_key, pad;
};
struct DevStats {
    unsigned long long lookups, hits, misses, evictions, trace_dropped;
    unsigned long long dev_fills;   // blobs copied by fill_kernel
};

struct MetaPtrs {
    LookupHdr* hdr;         // followed directly by MissEnt[E]
    MissEnt* miss;
    DevStats* stats;
    uint32_t* trace_count;
    int32_t* slot_table;    // [L*E]
    int32_t* key_of;        // [C]
    unsigned long long* stamp;  // [C]
    int32_t* slot_all;      // [E] slot of each requested expert of the last call
    int32_t* slot_hit;      // [E] hits only
    moe_trace_rec* trace;   // [trace_cap]
    const char** src_of;    // [L*E] device address of each key's mapped host blob (device fills)
};

struct MetaLayout {
    size_t hdr, stats, tcount, slot_table, key_of, stamp, slot_all, slot_hit, trace, src, bytes;
};

static MetaLayout meta_layout(const moe_shape* s, int C, int trace_cap)
{
    MetaLayout m{};
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    m.hdr = take(sizeof(LookupHdr) + sizeof(MissEnt) * (size_t)s->experts);
    m.stats = take(sizeof(DevStats));
    m.tcount = take(sizeof(uint32_t));
    m.slot_table = take(sizeof(int32_t) * (size_t)s->layers * s->experts);
    m.key_of = take(sizeof(int32_t) * (size_t)C);
    m.stamp = take(sizeof(unsigned long long) * (size_t)C);
    m.slot_all = take(sizeof(int32_t) * (size_t)s->experts);
    m.slot_hit = take(sizeof(int32_t) * (size_t)s->experts);
    m.trace = take(sizeof(moe_trace_rec) * (size_t)trace_cap);
    m.src = take(sizeof(void*) * (size_t)s->layers * s->experts);
    m.bytes = o;
    return m;
}

static MetaPtrs meta_ptrs(void* base, const MetaLayout& l)
{
    char* b = static_cast<char*>(base);
    MetaPtrs p;
    p.hdr = reinterpret_cast<LookupHdr*>(b + l.hdr);
    p.miss = reinterpret_cast<MissEnt*>(b + l.hdr + sizeof(LookupHdr));
    p.stats = reinterpret_cast<DevStats*>(b + l.stats);
    p.trace_count = reinterpret_cast<uint32_t*>(b + l.tcount);
    p.slot_table = reinterpret_cast<int32_t*>(b + l.slot_table);
    p.key_of = reinterpret_cast<int32_t*>(b + l.key_of);
    p.stamp = reinterpret_cast<unsigned long long*>(b + l.stamp);
    p.slot_all = reinterpret_cast<int32_t*>(b + l.slot_all);
    p.slot_hit = reinterpret_cast<int32_t*>(b + l.slot_hit);
    p.trace = reinterpret_cast<moe_trace_rec*>(b + l.trace);
    p.src_of = reinterpret_cast<const char**>(b + l.src);
    return p;
}

// -------------------------------------------------------------- block scan helper
// Exclusive prefix sum of one int per thread over a 1024-thread block.
__device__ int block_exclusive_scan(int v, int* s_warp, int* total)
{
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        int o = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += o;
    }
    if (lane == 31) s_warp[w] = inc;
    __syncthreads();
    if (w == 0) {
        int x = (lane < (blockDim.x >> 5)) ? s_warp[lane] : 0;
        int xi = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            int o = __shfl_up_sync(0xffffffffu, xi, off);
            if (lane >= off) xi += o;
        }
        s_warp[lane] = xi - x;           // exclusive warp offsets
        if (lane == 31) *total = xi;
    }
    __syncthreads();
    int r = s_warp[w] + inc - v;
    __syncthreads();
    return r;
}

__device__ __forceinline__ void put_rec(moe_trace_rec* tr, int cap, long pos, uint32_t call, int slot,
                                        int key, int E, int ev)
{
    if (pos < 0 || pos >= cap) return;
    moe_trace_rec r;
    r.call = call;
    r.slot = slot;
    r.layer = (uint16_t)(key / E);
    r.expert = (uint16_t)(key % E);
    r.event = (uint8_t)ev;
    r.pad[0] = r.pad[1] = r.pad[2] = 0;
    tr[pos] = r;
}

constexpr int kLookupThreads = 1024;

// Shared memory of one lookup: the layer's slot-table row, every slot's key
// and stamp, request flags, the miss list and its slots, victim flags.
static size_t lookup_smem_bytes(int E, int C)
{
    return align_up(sizeof(int) * E, 16) + align_up(sizeof(int) * C, 16) + align_up(8 * (size_t)C, 16) +
           align_up(E, 16) + align_up(sizeof(int) * E, 16) + align_up(sizeof(int) * E, 16) + align_up(C, 16);
}

// One CTA.  All state the call needs is read into shared memory in one
// parallel phase (one memory round trip), the decisions are made there,
// and only the entries that change are written back.
// The lookup, by every thread of a kLookupThreads CTA; smem: lookup_smem_bytes(E, C).
__device__ __forceinline__ void lookup_body(MetaPtrs m, int layer, const int32_t* __restrict__ idx, int count,
                                            int E, int C, int trace_cap, int32_t* __restrict__ slot_user,
                                            unsigned char* smem)
{
    unsigned char* p = smem;
    int* s_row = reinterpret_cast<int*>(p);                     p += align_up(sizeof(int) * E, 16);
    int* s_key = reinterpret_cast<int*>(p);                     p += align_up(sizeof(int) * C, 16);
    unsigned long long* s_stamp = reinterpret_cast<unsigned long long*>(p); p += align_up(8 * (size_t)C, 16);
    unsigned char* req = p;                                      p += align_up(E, 16);
    int* s_list = reinterpret_cast<int*>(p);                    p += align_up(sizeof(int) * E, 16);
    int* s_slot = reinterpret_cast<int*>(p);                    p += align_up(sizeof(int) * E, 16);
    unsigned char* s_cand = p;
    __shared__ int s_warp[32];
    __shared__ int s_tot, s_bad;
    __shared__ unsigned int s_base, s_clock;
    __shared__ unsigned long long s_wmin[32];
    const int tid = threadIdx.x;
    constexpr int NT = kLookupThreads;

    // ---- phase 0: everything in, in parallel
    for (int e = tid; e < E; e += NT) {
        req[e] = 0;
        s_row[e] = m.slot_table[layer * E + e];
    }
    for (int s = tid; s < C; s += NT) {
        s_key[s] = m.key_of[s];
        s_stamp[s] = m.stamp[s];
    }
    if (tid == 0) {
        s_bad = 0;
        s_base = *m.trace_count;
        s_clock = m.hdr->clock;
    }
    __syncthreads();
    for (int i = tid; i < count; i += NT) {
        int v = idx[i];
        if (v < 0 || v >= E) s_bad = 1;
        else req[v] = 1;
    }
    __syncthreads();
    LookupHdr* hdr = m.hdr;
    if (s_bad) {
        if (tid == 0) {
            hdr->status = MOE_ERR_INVALID_ARG;
            hdr->n_req = hdr->n_hit = hdr->n_miss = hdr->n_evict = 0;
            if (!hdr->sticky) hdr->sticky = MOE_ERR_INVALID_ARG;
        }
        for (int e = tid; e < E; e += NT) {
            m.slot_all[e] = m.slot_hit[e] = -1;
            if (slot_user) slot_user[e] = -1;
        }
        return;
    }
    // ---- classify: ranks of hits and misses in ascending expert id
    const int EPT = (E + NT - 1) / NT;
    const int e0 = tid * EPT;
    int nreq_loc = 0, nhit_loc = 0, nmiss_loc = 0;
    for (int e = e0; e < e0 + EPT && e < E; e++) {
        if (!req[e]) continue;
        nreq_loc++;
        if (s_row[e] >= 0) nhit_loc++;
        else nmiss_loc++;
    }
    block_exclusive_scan(nreq_loc, s_warp, &s_tot);
    const int nreq_tot = s_tot;
    __syncthreads();
    if (nreq_tot > C) {
        if (tid == 0) {
            hdr->status = MOE_ERR_CAPACITY;
            hdr->n_req = nreq_tot;
            hdr->n_hit = hdr->n_miss = hdr->n_evict = 0;
            if (!hdr->sticky) hdr->sticky = MOE_ERR_CAPACITY;
        }
        for (int e = tid; e < E; e += NT) {
            m.slot_all[e] = m.slot_hit[e] = -1;
            if (slot_user) slot_user[e] = -1;
        }
        return;
    }
    const int hit_base = block_exclusive_scan(nhit_loc, s_warp, &s_tot);
    const int nhit_tot = s_tot;
    __syncthreads();
    const int miss_base = block_exclusive_scan(nmiss_loc, s_warp, &s_tot);
    const int nmiss_tot = s_tot;
    __syncthreads();
    const unsigned long long T = (unsigned long long)s_clock + 1ull;
    const uint32_t base = s_base;

    // ---- hits: refresh stamps, records; list the misses
    {
        int hr = hit_base, mr = miss_base;
        for (int e = e0; e < e0 + EPT && e < E; e++) {
            if (!req[e]) {
                m.slot_all[e] = m.slot_hit[e] = -1;
                if (slot_user) slot_user[e] = -1;
                continue;
            }
            const int s = s_row[e];
            if (s >= 0) {
                s_stamp[s] = T;
                m.stamp[s] = T;
                put_rec(m.trace, trace_cap, (long)base + hr, (uint32_t)T, s, layer * E + e, E, MOE_EV_HIT);
                hr++;
                m.slot_all[e] = m.slot_hit[e] = s;
                if (slot_user) slot_user[e] = s;
            } else {
                s_list[mr++] = e;
            }
        }
    }
    // ---- free slots (ascending), victim candidates = resident keys not requested
    const int SPT = (C + NT - 1) / NT;
    const int s0 = tid * SPT;
    int nfree_loc = 0;
    for (int s = s0; s < s0 + SPT && s < C; s++) {
        const int k2 = s_key[s];
        const bool isfree = k2 < 0;
        nfree_loc += isfree;
        const bool in_r = !isfree && (k2 / E == layer) && req[k2 % E];
        s_cand[s] = (!isfree && !in_r) ? 1 : 0;
    }
    const int free_base = block_exclusive_scan(nfree_loc, s_warp, &s_tot);
    const int nfree = s_tot;
    __syncthreads();
    {
        int fr = free_base;
        for (int s = s0; s < s0 + SPT && s < C; s++) {
            if (s_key[s] < 0) {
                if (fr < nmiss_tot) s_slot[fr] = s;
                fr++;
            }
        }
    }
    // ---- victims: smallest (stamp, slot) among candidates, one block reduction each
    const int nvict = nmiss_tot > nfree ? nmiss_tot - nfree : 0;
    for (int r = 0; r < nvict; r++) {
        unsigned long long best = ~0ull;
        for (int s = s0; s < s0 + SPT && s < C; s++)
            if (s_cand[s]) {
                const unsigned long long key = (s_stamp[s] << 14) | (unsigned long long)s;
                best = key < best ? key : best;
            }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, best, off);
            best = o < best ? o : best;
        }
        if ((tid & 31) == 0) s_wmin[tid >> 5] = best;
        __syncthreads();
        if (tid < 32) {
            unsigned long long b = (tid < (NT >> 5)) ? s_wmin[tid] : ~0ull;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, b, off);
                b = o < b ? o : b;
            }
            if (tid == 0) {
                // a candidate always exists when |R| <= C; the guard keeps a
                // corrupted state from indexing out of range
                int vs = (b == ~0ull) ? 0 : (int)(b & 0x3FFFull);
                if (vs >= C) vs = 0;
                s_slot[nfree + r] = vs;
                s_cand[vs] = 0;
            }
        }
        __syncthreads();
    }
    __syncthreads();
    // ---- installs: miss i takes s_slot[i]
    for (int i = tid; i < nmiss_tot; i += NT) {
        const int e = s_list[i];
        const int key = layer * E + e;
        const int s = s_slot[i];
        long pos = (long)base + nhit_tot + i + (i > nfree ? i - nfree : 0);
        int old = -1;
        if (i >= nfree) {
            old = s_key[s];
            if (old >= 0) m.slot_table[old] = -1;
            put_rec(m.trace, trace_cap, pos, (uint32_t)T, s, old, E, MOE_EV_EVICT);
            pos++;
        }
        put_rec(m.trace, trace_cap, pos, (uint32_t)T, s, key, E, MOE_EV_MISS);
        MissEnt me;
        me.expert = e;
        me.slot = s;
        me.old_key = old;
        me.pad = 0;
        m.miss[i] = me;
        m.slot_table[key] = s;
        m.key_of[s] = key;
        m.stamp[s] = T;
        m.slot_all[e] = s;
        m.slot_hit[e] = -1;
        if (slot_user) slot_user[e] = s;
    }
    if (tid == 0) {
        const long total = (long)nhit_tot + nmiss_tot + nvict;
        long end = (long)base + total;
        if (end > trace_cap) {
            m.stats->trace_dropped += (unsigned long long)(end - ((long)base > (long)trace_cap ? (long)base : (long)trace_cap));
            end = trace_cap;
        }
        *m.trace_count = (uint32_t)(end > (long)base ? end : (long)base);
        hdr->status = MOE_OK;
        hdr->clock = (uint32_t)T;
        hdr->n_req = nreq_tot;
        hdr->n_hit = nhit_tot;
        hdr->n_miss = nmiss_tot;
        hdr->n_evict = nvict;
        hdr->n_free = nfree;
        m.stats->lookups += 1;
        m.stats->hits += nhit_tot;
        m.stats->misses += nmiss_tot;
        m.stats->evictions += nvict;
    }
}

__global__ void __launch_bounds__(kLookupThreads) lookup_kernel(MetaPtrs m, int layer,
                                                                const int32_t* __restrict__ idx,
                                                                int count, int E, int C, int trace_cap,
                                                                int32_t* __restrict__ slot_user)
{
    extern __shared__ __align__(16) unsigned char smem[];
    lookup_body(m, layer, idx, count, E, C, trace_cap, slot_user, smem);
}

// The front of a decode-sized layer call in one launch: top-k of the n <= 32
// tokens (a warp per token, from the logits the router kernel wrote), the
// lookup of their experts, and the token -> expert permutation; the same code
// as the separate router top-k, lookup and permutation kernels.
template <int EPL>
__global__ void __launch_bounds__(kLookupThreads) front_kernel(MetaPtrs m, int layer, const float* __restrict__ logits,
                                                               int n, int k, int E, int C, int trace_cap,
                                                               int32_t* __restrict__ idx, float* __restrict__ w,
                                                               int32_t* __restrict__ offsets,
                                                               int32_t* __restrict__ row_of,
                                                               int32_t* __restrict__ assign_of)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ PermSmem S;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp < n) topk_token<EPL>(logits + (size_t)warp * E, E, k, lane, idx + (size_t)warp * k, w + (size_t)warp * k);
    __syncthreads();   // the indices (global) are complete and visible to the whole CTA
    lookup_body(m, layer, idx, n * k, E, C, trace_cap, nullptr, smem);
    __syncthreads();
    perm_small_body(idx, n * k, E, offsets, row_of, assign_of, S);
}

// Undo the installs of a call whose fills could not be issued: the keys
// become non-resident and their slots free.  Victims stay evicted.
__global__ void rollback_kernel(MetaPtrs m, int n)
{
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        MissEnt me = m.miss[i];
        int key = m.key_of[me.slot];
        if (key >= 0) m.slot_table[key] = -1;
        m.key_of[me.slot] = -1;
        m.stamp[me.slot] = 0ull;
    }
}

constexpr int kFillCtas = 16;
constexpr int kFillThreads = 256;
constexpr int kFillUnroll = 8;   // 16-byte loads in flight per thread

// Device fills: copies the blobs on the miss list of the last lookup from
// mapped pinned host memory into their slots: the whole list (group < 0) or
// the misses of one miss group.  Runs after the lookup kernel in stream
// order and reads what it wrote; a failed lookup leaves nothing to copy.  The work is cut into rounds of kFillThreads * kFillUnroll 16-byte
// words (32 KiB) dealt out to the CTAs; every thread issues all its loads
// of a round before its stores, so 16 CTAs keep 512 KiB of PCIe reads in
// flight.  Blob and slot addresses are 16-byte aligned, slot_bytes is a
// multiple of 128.
__global__ void __launch_bounds__(kFillThreads) fill_kernel(MetaPtrs m, int layer, int E, char* __restrict__ pool,
                                                            size_t slot_bytes, int group)
{
    const LookupHdr* h = m.hdr;
    if (h->status != MOE_OK) return;
    const int nm = h->n_miss;
    int i0 = 0, i1 = nm;
    if (group >= 0) miss_group(nm, group, &i0, &i1);
    if (i1 <= i0) return;
    constexpr size_t kRound = (size_t)kFillThreads * kFillUnroll;
    const size_t n16 = slot_bytes / 16;
    const size_t rounds = (n16 + kRound - 1) / kRound;
    const size_t total = rounds * (size_t)(i1 - i0);
    for (size_t p = blockIdx.x; p < total; p += gridDim.x) {
        const int i = i0 + (int)(p / rounds);
        const size_t b = (p - (size_t)(i - i0) * rounds) * kRound + threadIdx.x;
        const MissEnt me = m.miss[i];
        const int4* __restrict__ src = reinterpret_cast<const int4*>(m.src_of[(size_t)layer * E + me.expert]);
        int4* __restrict__ dst = reinterpret_cast<int4*>(pool + (size_t)me.slot * slot_bytes);
        int4 v[kFillUnroll];
#pragma unroll
        for (int u = 0; u < kFillUnroll; u++) {
            const size_t w = b + (size_t)u * kFillThreads;
            if (w < n16) v[u] = src[w];
        }
#pragma unroll
        for (int u = 0; u < kFillUnroll; u++) {
            const size_t w = b + (size_t)u * kFillThreads;
            if (w < n16) dst[w] = v[u];
        }
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) m.stats->dev_fills += (unsigned long long)(i1 - i0);
}

// Slot tables of the miss groups of the last lookup: out[g][e] is the slot
// of expert e when e is a miss of group g, else -1.  A failed lookup leaves
// every entry -1.
__global__ void group_slots_kernel(MetaPtrs m, int E, int32_t* __restrict__ out)
{
    for (int i = threadIdx.x; i < kMissGroups * E; i += blockDim.x) out[i] = -1;
    __syncthreads();
    const int nm = m.hdr->status == MOE_OK ? m.hdr->n_miss : 0;
    for (int g = 0; g < kMissGroups; g++) {
        int b, e;
        miss_group(nm, g, &b, &e);
        for (int i = b + threadIdx.x; i < e; i += blockDim.x) {
            const MissEnt me = m.miss[i];
            if (me.expert >= 0 && me.expert < E) out[g * E + me.expert] = me.slot;
        }
    }
}

}  // namespace moe

// ====================================================================== host side
struct moe_cache {
    moe_shape shape;
    int C;
    int trace_cap;
    size_t slot_bytes;
    void* d_meta;
    moe::MetaLayout ml;
    moe::MetaPtrs m;
    char* pool;
    std::vector<const void*> blobs;
    std::vector<const char*> dsrc;       // device addresses of the blobs (device fills)
    int fill_mode = MOE_FILL_HOST;
    std::vector<int> resident;           // host mirror: resident keys per layer
    std::vector<unsigned char> hbuf;     // LookupHdr + MissEnt[E]
    cudaEvent_t ev_lookup = nullptr, ev_fill = nullptr;
    cudaEvent_t ev_pf[2] = {nullptr, nullptr};   // fills of the two layers a prefill has in flight
    cudaEvent_t ev_grp[moe::kMissGroups] = {};         // fills of each miss group of a layer call
    uint64_t fill_bytes = 0, host_syncs = 0, fills_issued = 0;
    long fault_fill_at = 0;              // MOE_FAULT_INJECT=fill_fail:<n>
    int lookup_smem = 0;
    int front_smem_set = 0;   // dynamic shared memory the front kernels are allowed (per cache)
};

namespace moe {


// Enqueue the lookup kernel for `layer`.
int cache_launch_lookup(moe_cache* c, int layer, const int32_t* idx, int count, int32_t* slot_user,
                        cudaStream_t st)
{
    {
        ProfScope ps(MOE_PROF_LOOKUP, st);
        prof_count(MOE_PROF_LOOKUP, 1);
        lookup_kernel<<<1, kLookupThreads, c->lookup_smem, st>>>(c->m, layer, idx, count, c->shape.experts,
                                                             c->C, c->trace_cap, slot_user);
        MOE_LAUNCH_CHECK();
    }
    // everything before this point on `st` (earlier readers of any victim
    // slot included) is complete once ev_lookup fires
    MOE_CUDA_TRY(cudaEventRecord(c->ev_lookup, st));
    return MOE_OK;
}

// Whether a call of n tokens is small enough for the fused front kernel.
bool cache_front_fits(const moe_cache* c, int n)
{
    const int E = c->shape.experts, k = c->shape.top_k;
    return n > 0 && n <= kLookupThreads / 32 && E <= 1024 && n * k <= kSmallA && E <= kSmallE;
}

// The fused front (top-k + lookup + permutation) for n tokens, when
// cache_front_fits; MOE_ERR_UNSUPPORTED otherwise (nothing enqueued).
int cache_launch_front(moe_cache* c, int layer, const float* logits, int n, int32_t* idx, float* w,
                       int32_t* offsets, int32_t* row_of, int32_t* assign_of, cudaStream_t st)
{
    const int E = c->shape.experts, k = c->shape.top_k;
    if (!cache_front_fits(c, n)) return MOE_ERR_UNSUPPORTED;
    if (c->front_smem_set < c->lookup_smem) {
        if (c->lookup_smem > 48 * 1024) {
            MOE_CUDA_TRY(cudaFuncSetAttribute(front_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, c->lookup_smem));
            MOE_CUDA_TRY(cudaFuncSetAttribute(front_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, c->lookup_smem));
        }
        c->front_smem_set = c->lookup_smem;
    }
    {
        ProfScope ps(MOE_PROF_LOOKUP, st);
        prof_count(MOE_PROF_LOOKUP, 1);
        if (E <= 256)
            front_kernel<8><<<1, kLookupThreads, c->lookup_smem, st>>>(c->m, layer, logits, n, k, E, c->C, c->trace_cap,
                                                                       idx, w, offsets, row_of, assign_of);
        else
            front_kernel<32><<<1, kLookupThreads, c->lookup_smem, st>>>(c->m, layer, logits, n, k, E, c->C,
                                                                        c->trace_cap, idx, w, offsets, row_of,
                                                                        assign_of);
        MOE_LAUNCH_CHECK();
    }
    MOE_CUDA_TRY(cudaEventRecord(c->ev_lookup, st));
    return MOE_OK;
}

bool cache_layer_resident(const moe_cache* c, int layer) { return c->resident[layer] == c->shape.experts; }

const int32_t* cache_slot_all(const moe_cache* c) { return c->m.slot_all; }
const int32_t* cache_slot_hit(const moe_cache* c) { return c->m.slot_hit; }
const char* cache_pool(const moe_cache* c) { return c->pool; }
size_t cache_slot_bytes(const moe_cache* c) { return c->slot_bytes; }

// Host side of a lookup that may miss: wait for the lookup kernel, read the
// miss list, issue one copy per miss on `copy` after everything before the
// lookup on the compute stream is done, and record `ev` (ev_fill by
// default).  *n_miss gets the number of fills issued; the caller makes the
// compute stream wait on the event when *n_miss > 0.
int cache_read_and_fill(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, int* n_miss, cudaEvent_t ev,
                        bool groups)
{
    if (!ev) ev = c->ev_fill;
    *n_miss = 0;
    const int E = c->shape.experts;
    // one read-back of the header and the whole miss list, ordered after the
    // lookup kernel through ev_lookup (not after later work on `st`)
    MOE_CUDA_TRY(cudaStreamWaitEvent(copy, c->ev_lookup, 0));
    MOE_CUDA_TRY(cudaMemcpyAsync(c->hbuf.data(), c->m.hdr, c->hbuf.size(), cudaMemcpyDeviceToHost, copy));
    MOE_CUDA_TRY(cudaStreamSynchronize(copy));
    c->host_syncs++;
    const LookupHdr* h = reinterpret_cast<const LookupHdr*>(c->hbuf.data());
    if (h->status != MOE_OK) return h->status;
    if (h->n_miss == 0) return MOE_OK;
    const MissEnt* ms = reinterpret_cast<const MissEnt*>(c->hbuf.data() + sizeof(LookupHdr));
    // mirror: evictions leave
    for (int i = 0; i < h->n_miss; i++)
        if (ms[i].old_key >= 0) c->resident[ms[i].old_key / E]--;
    bool fail = c->fault_fill_at > 0 && c->fills_issued < (uint64_t)c->fault_fill_at &&
                c->fills_issued + (uint64_t)h->n_miss >= (uint64_t)c->fault_fill_at;
    if (fail) {
        // injected failure before any copy: undo this call's installs
        c->fault_fill_at = 0;
        rollback_kernel<<<1, 256, 0, st>>>(c->m, h->n_miss);
        MOE_LAUNCH_CHECK();
        MOE_CUDA_TRY(cudaStreamSynchronize(st));
        return MOE_ERR_FILL;
    }
    ProfScope ps(MOE_PROF_FILL, copy);
    prof_count(MOE_PROF_FILL, h->n_miss);
    // in miss-list order; with groups, each non-empty group's copies are
    // followed by its event
    for (int g = 0; g < (groups ? kMissGroups : 1); g++) {
        int b = 0, e = h->n_miss;
        if (groups) miss_group(h->n_miss, g, &b, &e);
        for (int i = b; i < e; i++) {
            const void* src = c->blobs[(size_t)layer * E + ms[i].expert];
            if (!src) return MOE_ERR_STATE;
            MOE_CUDA_TRY(cudaMemcpyAsync(c->pool + (size_t)ms[i].slot * c->slot_bytes, src, c->slot_bytes,
                                         cudaMemcpyHostToDevice, copy));
            c->resident[layer]++;
        }
        if (groups && e > b) MOE_CUDA_TRY(cudaEventRecord(c->ev_grp[g], copy));
    }
    c->fills_issued += (uint64_t)h->n_miss;
    c->fill_bytes += (uint64_t)h->n_miss * c->slot_bytes;
    MOE_CUDA_TRY(cudaEventRecord(ev, copy));
    *n_miss = h->n_miss;
    return MOE_OK;
}

int cache_fill_mode(const moe_cache* c) { return c->fill_mode; }

// Device fills of the last lookup on `layer` (all misses, or miss group
// `group`): the copy stream waits for the lookup (and so for every earlier
// reader of a victim slot on the compute stream), runs fill_kernel and
// records ev (ev_fill by default).  Nothing is read back.
int cache_launch_device_fill(moe_cache* c, int layer, cudaStream_t copy, cudaEvent_t ev, int group)
{
    if (!ev) ev = c->ev_fill;
    MOE_CUDA_TRY(cudaStreamWaitEvent(copy, c->ev_lookup, 0));
    {
        ProfScope ps(MOE_PROF_FILL, copy);
        prof_count(MOE_PROF_FILL, 1);
        fill_kernel<<<kFillCtas, kFillThreads, 0, copy>>>(c->m, layer, c->shape.experts, c->pool, c->slot_bytes,
                                                          group);
        MOE_LAUNCH_CHECK();
    }
    MOE_CUDA_TRY(cudaEventRecord(ev, copy));
    return MOE_OK;
}

// The fills of the lookup just enqueued for `layer`, as miss groups: group
// g's slots have landed once cache_group_event(c, g) fires.  *live gets the
// groups that may hold misses: with device fills all of them (the miss list
// stays on the device; an empty group's kernel copies nothing), with host
// fills the non-empty ones (the host reads the miss list back).
int cache_group_fills(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, unsigned* live)
{
    *live = 0;
    if (c->fill_mode == MOE_FILL_DEVICE) {
        for (int g = 0; g < kMissGroups; g++) {
            int rc = cache_launch_device_fill(c, layer, copy, c->ev_grp[g], g);
            if (rc) return rc;
        }
        *live = (1u << kMissGroups) - 1;
        return MOE_OK;
    }
    int nm = 0;
    int rc = cache_read_and_fill(c, layer, st, copy, &nm, nullptr, true);
    if (rc) return rc;
    for (int g = 0; g < kMissGroups; g++) {
        int b, e;
        miss_group(nm, g, &b, &e);
        if (e > b) *live |= 1u << g;
    }
    return MOE_OK;
}

// group_slots_kernel for the last lookup, on `st`: grp_slots [kMissGroups][E].
int cache_launch_group_slots(moe_cache* c, int32_t* grp_slots, cudaStream_t st)
{
    ProfScope ps(MOE_PROF_LOOKUP, st);
    prof_count(MOE_PROF_LOOKUP, 1);
    group_slots_kernel<<<1, 256, 0, st>>>(c->m, c->shape.experts, grp_slots);
    MOE_LAUNCH_CHECK();
    return MOE_OK;
}

cudaEvent_t cache_group_event(const moe_cache* c, int g) { return c->ev_grp[g]; }

// The fills of the lookup just enqueued on `st` for `layer`, whichever fill
// mode the cache is in; `ev` completes once they have landed (recorded on
// `st` itself when there is nothing to copy), so work that waits on it sees
// every slot of the lookup filled.
int cache_fill(moe_cache* c, int layer, cudaStream_t st, cudaStream_t copy, cudaEvent_t ev)
{
    if (c->fill_mode == MOE_FILL_DEVICE) return cache_launch_device_fill(c, layer, copy, ev);
    int nm = 0;
    if (!cache_layer_resident(c, layer)) {
        int rc = cache_read_and_fill(c, layer, st, copy, &nm, ev);
        if (rc) return rc;
    }
    if (nm == 0) MOE_CUDA_TRY(cudaEventRecord(ev, st));
    return MOE_OK;
}

cudaEvent_t cache_prefill_event(const moe_cache* c, int i) { return c->ev_pf[i & 1]; }

// Host mirror of the resident keys per layer, recounted from the slot table.
static int resync_resident(moe_cache* c, cudaStream_t st)
{
    const int E = c->shape.experts;
    const size_t nkeys = (size_t)c->shape.layers * E;
    std::vector<int32_t> table(nkeys);
    MOE_CUDA_TRY(cudaStreamSynchronize(st));
    MOE_CUDA_TRY(cudaMemcpy(table.data(), c->m.slot_table, 4 * nkeys, cudaMemcpyDeviceToHost));
    c->resident.assign(c->shape.layers, 0);
    for (size_t k = 0; k < nkeys; k++)
        if (table[k] >= 0) c->resident[k / E]++;
    return MOE_OK;
}

const moe_shape* cache_shape(const moe_cache* c) { return &c->shape; }

int cache_capacity_int(const moe_cache* c) { return c->C; }

}  // namespace moe

using namespace moe;

extern "C" size_t moe_cache_meta_bytes(const moe_shape* shape, int32_t capacity, int32_t trace_capacity)
{
    if (!shape_ok(shape) || capacity <= 0 || capacity > kMaxCapacity || trace_capacity < 0) return 0;
    return meta_layout(shape, capacity, trace_capacity).bytes;
}

extern "C" int moe_cache_create(const moe_shape* shape, void* d_meta, size_t meta_bytes, void* d_slot_pool,
                                int32_t capacity, int32_t trace_capacity, const void* const* h_blobs,
                                void* stream, moe_cache** out)
{
    if (!out) return MOE_ERR_INVALID_ARG;
    *out = nullptr;
    if (!shape_ok(shape) || capacity <= 0 || capacity > kMaxCapacity || trace_capacity < 0 || !d_meta ||
        !d_slot_pool || !h_blobs)
        return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_meta | (uintptr_t)d_slot_pool) & 255) return MOE_ERR_INVALID_ARG;
    MetaLayout ml = meta_layout(shape, capacity, trace_capacity);
    if (meta_bytes < ml.bytes) return MOE_ERR_INVALID_ARG;
    moe_cache* c = new moe_cache();
    c->shape = *shape;
    c->C = capacity;
    c->trace_cap = trace_capacity;
    c->slot_bytes = blob_layout(shape).bytes;
    c->d_meta = d_meta;
    c->ml = ml;
    c->m = meta_ptrs(d_meta, ml);
    c->pool = static_cast<char*>(d_slot_pool);
    size_t nkeys = (size_t)shape->layers * shape->experts;
    c->blobs.assign(h_blobs, h_blobs + nkeys);
    c->resident.assign(shape->layers, 0);
    c->hbuf.resize(sizeof(LookupHdr) + sizeof(MissEnt) * (size_t)shape->experts);
    c->lookup_smem = (int)lookup_smem_bytes(shape->experts, capacity);
    if (const char* fi = getenv("MOE_FAULT_INJECT")) {
        if (!strncmp(fi, "fill_fail:", 10)) c->fault_fill_at = atol(fi + 10);
    }
    cudaStream_t st = as_stream(stream);
    auto fail = [&](int rc) { moe_cache_destroy(c); return rc; };
    if (cudaEventCreateWithFlags(&c->ev_lookup, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_fill, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_pf[0], cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&c->ev_pf[1], cudaEventDisableTiming) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    for (cudaEvent_t& e : c->ev_grp)
        if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return fail(MOE_ERR_CUDA);
    if (c->lookup_smem > 48 * 1024 &&
        cudaFuncSetAttribute(lookup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, c->lookup_smem) !=
            cudaSuccess)
        return fail(MOE_ERR_CUDA);
    // zero everything, then mark every slot table entry and slot key empty
    std::vector<int32_t> neg((size_t)std::max<size_t>(nkeys, (size_t)capacity), -1);
    if (cudaMemsetAsync(d_meta, 0, ml.bytes, st) != cudaSuccess ||
        cudaMemcpyAsync(c->m.slot_table, neg.data(), sizeof(int32_t) * nkeys, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaMemcpyAsync(c->m.key_of, neg.data(), sizeof(int32_t) * capacity, cudaMemcpyHostToDevice, st) !=
            cudaSuccess ||
        cudaStreamSynchronize(st) != cudaSuccess)
        return fail(MOE_ERR_CUDA);
    *out = c;
    return MOE_OK;
}

extern "C" int moe_cache_destroy(moe_cache* c)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    if (c->ev_lookup) cudaEventDestroy(c->ev_lookup);
    if (c->ev_fill) cudaEventDestroy(c->ev_fill);
    for (cudaEvent_t e : c->ev_pf)
        if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : c->ev_grp)
        if (e) cudaEventDestroy(e);
    delete c;
    return MOE_OK;
}

extern "C" int32_t moe_cache_capacity(const moe_cache* c) { return c ? c->C : 0; }

extern "C" int moe_cache_lookup_update(moe_cache* c, int32_t layer, const int32_t* d_idx, int32_t count,
                                       int32_t* d_slot_of_expert, void* stream, void* copy_stream)
{
    if (!c || layer < 0 || layer >= c->shape.layers || count < 0 || (count > 0 && !d_idx))
        return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream), cp = as_stream(copy_stream);
    int rc = cache_launch_lookup(c, layer, d_idx, count, d_slot_of_expert, st);
    if (rc) return rc;
    if (c->fill_mode == MOE_FILL_DEVICE) {
        if ((rc = cache_launch_device_fill(c, layer, cp))) return rc;
        MOE_CUDA_TRY(cudaStreamWaitEvent(st, c->ev_fill, 0));
        return MOE_OK;
    }
    if (cache_layer_resident(c, layer)) return MOE_OK;
    int nm = 0;
    rc = cache_read_and_fill(c, layer, st, cp, &nm);
    if (rc) return rc;
    if (nm > 0) MOE_CUDA_TRY(cudaStreamWaitEvent(st, c->ev_fill, 0));
    return MOE_OK;
}

extern "C" int moe_cache_read_trace(moe_cache* c, moe_trace_rec* h_buf, size_t cap, size_t* n_out)
{
    if (!c || !n_out || (cap && !h_buf)) return MOE_ERR_INVALID_ARG;
    *n_out = 0;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    uint32_t n = 0;
    MOE_CUDA_TRY(cudaMemcpy(&n, c->m.trace_count, sizeof n, cudaMemcpyDeviceToHost));
    size_t take = std::min<size_t>(n, cap);
    if (take) MOE_CUDA_TRY(cudaMemcpy(h_buf, c->m.trace, take * sizeof(moe_trace_rec), cudaMemcpyDeviceToHost));
    uint32_t zero = 0;
    MOE_CUDA_TRY(cudaMemcpy(c->m.trace_count, &zero, sizeof zero, cudaMemcpyHostToDevice));
    *n_out = take;
    return MOE_OK;
}

extern "C" int moe_cache_get_stats(moe_cache* c, moe_cache_stats* out)
{
    if (!c || !out) return MOE_ERR_INVALID_ARG;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    DevStats d;
    MOE_CUDA_TRY(cudaMemcpy(&d, c->m.stats, sizeof d, cudaMemcpyDeviceToHost));
    out->lookups = d.lookups;
    out->hits = d.hits;
    out->misses = d.misses;
    out->evictions = d.evictions;
    out->trace_dropped = d.trace_dropped;
    out->fill_bytes = c->fill_bytes + d.dev_fills * (uint64_t)c->slot_bytes;
    out->host_syncs = c->host_syncs;
    return MOE_OK;
}

extern "C" int moe_cache_snapshot(moe_cache* c, int32_t* h_slot_of, int32_t* h_key_of, uint64_t* h_stamp)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    size_t nkeys = (size_t)c->shape.layers * c->shape.experts;
    if (h_slot_of) MOE_CUDA_TRY(cudaMemcpy(h_slot_of, c->m.slot_table, 4 * nkeys, cudaMemcpyDeviceToHost));
    if (h_key_of) MOE_CUDA_TRY(cudaMemcpy(h_key_of, c->m.key_of, 4 * (size_t)c->C, cudaMemcpyDeviceToHost));
    if (h_stamp) MOE_CUDA_TRY(cudaMemcpy(h_stamp, c->m.stamp, 8 * (size_t)c->C, cudaMemcpyDeviceToHost));
    return MOE_OK;
}

// Resize at a safe point.  Host logic over a synchronous snapshot of the
// bookkeeping: evict the surplus by (last use, slot), pack the survivors to
// the front in old-slot order, copy their blobs device to device, write the
// new bookkeeping.
extern "C" int moe_cache_resize(moe_cache* c, void* d_meta_new, size_t meta_bytes, void* d_pool_new,
                                int32_t new_capacity, void* stream)
{
    if (!c || !d_meta_new || !d_pool_new || new_capacity <= 0 || new_capacity > kMaxCapacity)
        return MOE_ERR_INVALID_ARG;
    if (((uintptr_t)d_meta_new | (uintptr_t)d_pool_new) & 255) return MOE_ERR_INVALID_ARG;
    MetaLayout nl = meta_layout(&c->shape, new_capacity, c->trace_cap);
    if (meta_bytes < nl.bytes) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    MOE_CUDA_TRY(cudaStreamSynchronize(st));
    // device fills leave the host mirror stale: recount it first
    if (c->fill_mode == MOE_FILL_DEVICE) {
        int rc = resync_resident(c, st);
        if (rc) return rc;
    }
    const int E = c->shape.experts, C = c->C;
    const size_t nkeys = (size_t)c->shape.layers * E;
    std::vector<int32_t> table(nkeys), key(C);
    std::vector<unsigned long long> stamp(C);
    LookupHdr hdr;
    DevStats stats;
    uint32_t tcount = 0;
    MOE_CUDA_TRY(cudaMemcpy(table.data(), c->m.slot_table, 4 * nkeys, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(key.data(), c->m.key_of, 4 * (size_t)C, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(stamp.data(), c->m.stamp, 8 * (size_t)C, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(&hdr, c->m.hdr, sizeof hdr, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(&stats, c->m.stats, sizeof stats, cudaMemcpyDeviceToHost));
    MOE_CUDA_TRY(cudaMemcpy(&tcount, c->m.trace_count, 4, cudaMemcpyDeviceToHost));
    std::vector<moe_trace_rec> recs(tcount);
    if (tcount)
        MOE_CUDA_TRY(cudaMemcpy(recs.data(), c->m.trace, sizeof(moe_trace_rec) * tcount, cudaMemcpyDeviceToHost));
    const uint32_t clock = hdr.clock;
    auto rec = [&](int slot, int k, int ev) {
        moe_trace_rec r{};
        r.call = clock;
        r.slot = slot;
        r.layer = (uint16_t)(k / E);
        r.expert = (uint16_t)(k % E);
        r.event = (uint8_t)ev;
        recs.push_back(r);
    };
    // surplus eviction by (stamp, slot)
    std::vector<int> live;
    for (int s = 0; s < C; s++)
        if (key[s] >= 0) live.push_back(s);
    std::vector<int> by_age = live;
    std::sort(by_age.begin(), by_age.end(), [&](int a, int b) {
        return stamp[a] != stamp[b] ? stamp[a] < stamp[b] : a < b;
    });
    size_t surplus = live.size() > (size_t)new_capacity ? live.size() - new_capacity : 0;
    for (size_t i = 0; i < surplus; i++) {
        int s = by_age[i];
        rec(s, key[s], MOE_EV_EVICT);
        table[key[s]] = -1;
        c->resident[key[s] / E]--;
        key[s] = -1;
        stats.evictions++;
    }
    // pack survivors in old-slot order
    std::vector<int32_t> nkey(new_capacity, -1);
    std::vector<unsigned long long> nstamp(new_capacity, 0ull);
    int mnew = 0;
    const bool same_pool = d_pool_new == c->pool;
    for (int s = 0; s < C; s++) {
        if (key[s] < 0) continue;
        nkey[mnew] = key[s];
        nstamp[mnew] = stamp[s];
        table[key[s]] = mnew;
        if (mnew != s) rec(mnew, key[s], MOE_EV_MOVE);
        if (mnew != s || !same_pool)
            MOE_CUDA_TRY(cudaMemcpyAsync(static_cast<char*>(d_pool_new) + (size_t)mnew * c->slot_bytes,
                                         c->pool + (size_t)s * c->slot_bytes, c->slot_bytes,
                                         cudaMemcpyDeviceToDevice, st));
        mnew++;
    }
    MOE_CUDA_TRY(cudaStreamSynchronize(st));
    // new bookkeeping
    MetaPtrs nm = meta_ptrs(d_meta_new, nl);
    if (recs.size() > (size_t)c->trace_cap) {
        stats.trace_dropped += recs.size() - c->trace_cap;
        recs.resize(c->trace_cap);
    }
    uint32_t ntc = (uint32_t)recs.size();
    std::vector<unsigned char> hb(sizeof(LookupHdr), 0);
    LookupHdr nh{};
    nh.status = MOE_OK;
    nh.clock = clock;
    nh.sticky = hdr.sticky;
    MOE_CUDA_TRY(cudaMemsetAsync(d_meta_new, 0, nl.bytes, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.hdr, &nh, sizeof nh, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.stats, &stats, sizeof stats, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.trace_count, &ntc, 4, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.slot_table, table.data(), 4 * nkeys, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.key_of, nkey.data(), 4 * (size_t)new_capacity, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaMemcpyAsync(nm.stamp, nstamp.data(), 8 * (size_t)new_capacity, cudaMemcpyHostToDevice, st));
    if (ntc)
        MOE_CUDA_TRY(cudaMemcpyAsync(nm.trace, recs.data(), sizeof(moe_trace_rec) * ntc, cudaMemcpyHostToDevice, st));
    if (!c->dsrc.empty())
        MOE_CUDA_TRY(cudaMemcpyAsync(nm.src_of, c->dsrc.data(), sizeof(void*) * nkeys, cudaMemcpyHostToDevice, st));
    MOE_CUDA_TRY(cudaStreamSynchronize(st));
    c->C = new_capacity;
    c->d_meta = d_meta_new;
    c->ml = nl;
    c->m = nm;
    c->pool = static_cast<char*>(d_pool_new);
    c->lookup_smem = (int)lookup_smem_bytes(E, new_capacity);
    if (c->lookup_smem > 48 * 1024)
        MOE_CUDA_TRY(cudaFuncSetAttribute(lookup_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, c->lookup_smem));
    return MOE_OK;
}

extern "C" int moe_cache_set_fill_mode(moe_cache* c, int32_t mode, void* stream)
{
    if (!c || (mode != MOE_FILL_HOST && mode != MOE_FILL_DEVICE)) return MOE_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    MOE_CUDA_TRY(cudaStreamSynchronize(st));
    if (mode == MOE_FILL_DEVICE) {
        const size_t nkeys = c->blobs.size();
        std::vector<const char*> d(nkeys);
        const void* last = nullptr;
        const char* last_d = nullptr;
        for (size_t k = 0; k < nkeys; k++) {
            const char* b = static_cast<const char*>(c->blobs[k]);
            if (b && b == last) { d[k] = last_d; continue; }   // keys often share a blob
            if (!b || ((uintptr_t)b & 15)) return MOE_ERR_INVALID_ARG;
            // both ends of the blob must be mapped host memory of one mapping
            cudaPointerAttributes a0, a1;
            if (cudaPointerGetAttributes(&a0, b) != cudaSuccess ||
                cudaPointerGetAttributes(&a1, b + c->slot_bytes - 1) != cudaSuccess) {
                cudaGetLastError();
                return MOE_ERR_INVALID_ARG;
            }
            if (a0.type != cudaMemoryTypeHost || a1.type != cudaMemoryTypeHost || !a0.devicePointer ||
                static_cast<const char*>(a1.devicePointer) !=
                    static_cast<const char*>(a0.devicePointer) + c->slot_bytes - 1)
                return MOE_ERR_INVALID_ARG;
            last = b;
            last_d = static_cast<const char*>(a0.devicePointer);
            d[k] = last_d;
        }
        // The fill kernel runs beside the FFN kernels, whose CTAs need nearly
        // all of an SM's shared memory.  An SM configures its L1 / shared
        // split for the kernel it runs; the fill CTAs ask for the largest
        // shared share so that FFN CTAs can join them on the same SMs.
        MOE_CUDA_TRY(cudaFuncSetAttribute(fill_kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                          (int)cudaSharedmemCarveoutMaxShared));
        MOE_CUDA_TRY(cudaMemcpyAsync(c->m.src_of, d.data(), sizeof(void*) * nkeys, cudaMemcpyHostToDevice, st));
        MOE_CUDA_TRY(cudaStreamSynchronize(st));
        c->dsrc.swap(d);
    } else if (c->fill_mode == MOE_FILL_DEVICE) {
        int rc = resync_resident(c, st);
        if (rc) return rc;
    }
    c->fill_mode = mode;
    return MOE_OK;
}

extern "C" int32_t moe_cache_fill_mode(const moe_cache* c) { return c ? c->fill_mode : MOE_ERR_INVALID_ARG; }

extern "C" int moe_cache_device_status(moe_cache* c, int32_t clear)
{
    if (!c) return MOE_ERR_INVALID_ARG;
    MOE_CUDA_TRY(cudaDeviceSynchronize());
    int32_t sticky = 0;
    MOE_CUDA_TRY(cudaMemcpy(&sticky, &c->m.hdr->sticky, sizeof sticky, cudaMemcpyDeviceToHost));
    if (clear && sticky) {
        const int32_t zero = 0;
        MOE_CUDA_TRY(cudaMemcpy(&c->m.hdr->sticky, &zero, sizeof zero, cudaMemcpyHostToDevice));
    }
    return sticky;
}
