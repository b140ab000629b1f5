/*
 * CPU oracle for the routed MoE layer with a GPU expert-slot cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, single-threaded,
 * obviously-correct statement of what the layer computes.  Only the tests,
 * the package's smoke check and the benchmark's CPU-baseline leg may load
 * it.  It shares no code, header, table or constant with the CUDA library,
 * and the CUDA library never calls it.
 *
 * Sources (FreeToken web pages, cited by page title and section):
 *  - routing of each token to a few of many experts: "FreeToken linux",
 *    section "Como gestiona FreeToken la memoria MoE" (6 of 256 routed
 *    experts per layer for DeepSeek-V4-Flash);
 *  - one LRU expert cache shared by all MoE layers, entries are whole
 *    (layer, expert) pairs, misses are brought into GPU slots: same section,
 *    and "FreeToken rtx 4090", section "Como funciona la jerarquia de memoria
 *    MoE";
 *  - elastic resize of that cache: "FreeToken quantization", section
 *    "Flujo de configuracion de la cuantizacion de FreeToken";
 *  - MXFP4 / NVFP4 / BF16 expert weights: "FreeToken quantization", sections
 *    "La cuantizacion de FreeToken y el modelo de servicio principal" and
 *    "Formatos compatibles, hardware y perfil de rendimiento".
 * The pages give no formulas.  Where they are silent this file takes the
 * readings listed in the repository design notes: softmax over the router
 * logits then top-k renormalised; SwiGLU experts; E2M1/E8M0/E4M3 as in the
 * OCP Microscaling v1.0 and NVIDIA NVFP4 public format descriptions; the
 * LRU tie and resize rules stated below.
 *
 * Arithmetic: fp64 accumulation everywhere, except the router logits, which
 * decide integer outputs (the top-k indices) and are therefore formed in the
 * kernel's precision and order (fp32 fused multiply-adds, lane-chunk order,
 * xor-butterfly across 32 lanes), written out here as a plain loop.
 *
 * Parity pins (tests): brute-force top-k and a library softmax for the
 * router; torch's float8 decoders and the OCP E2M1 table for the formats;
 * an OrderedDict simulator plus invariants for the LRU; numpy's stable
 * argsort for the permutation; hand-computed tiny layers for the FFN and
 * combine.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_CAPACITY (-2)

/* ------------------------------------------------------------------ */
/* number formats                                                      */
/* ------------------------------------------------------------------ */

/* E2M1: 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.
 * e == 0 is the subnormal range: value m * 0.5. */
double orc_e2m1(int code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* E8M0: unsigned power of two 2^(c-127); 255 encodes NaN. */
double orc_e8m0(int code)
{
    if (code == 255) return NAN;
    return ldexp(1.0, code - 127);
}

/* E4M3 (no infinities): 1 sign, 4 exponent bits (bias 7), 3 mantissa
 * bits; S.1111.111 is NaN; e == 0 gives subnormals m/8 * 2^-6. */
double orc_e4m3(int code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp(m / 8.0, -6);
    else mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Element (r, c) of a [rows][cols] matrix of packed E2M1 codes, two per
 * byte along a row, the even column in the low nibble. */
static int fp4_code(const uint8_t* q, int cols, int r, int c)
{
    uint8_t byte = q[(size_t)r * (cols / 2) + c / 2];
    return (c & 1) ? (byte >> 4) : (byte & 15);
}

/* MXFP4 -> real: w = e2m1 * 2^(scale-127), one E8M0 scale per 32 elements
 * along a row. */
void orc_dequant_mxfp4(const uint8_t* q, const uint8_t* sc, int rows, int cols, double* out)
{
    double v[16], s[256];  /* the decoders above, tabulated once */
    for (int i = 0; i < 16; i++) v[i] = orc_e2m1(i);
    for (int i = 0; i < 256; i++) s[i] = orc_e8m0(i);
    for (int r = 0; r < rows; r++)
        for (int c = 0; c < cols; c++)
            out[(size_t)r * cols + c] = v[fp4_code(q, cols, r, c)] * s[sc[(size_t)r * (cols / 32) + c / 32]];
}

/* NVFP4 -> real: w = e2m1 * e4m3(scale) * s_tensor, one E4M3 scale per 16
 * elements along a row, one fp32 scale for the whole matrix. */
void orc_dequant_nvfp4(const uint8_t* q, const uint8_t* sc, float s_tensor, int rows, int cols,
                       double* out)
{
    double v[16], s[256];  /* the decoders above, tabulated once */
    for (int i = 0; i < 16; i++) v[i] = orc_e2m1(i);
    for (int i = 0; i < 256; i++) s[i] = orc_e4m3(i);
    for (int r = 0; r < rows; r++)
        for (int c = 0; c < cols; c++)
            out[(size_t)r * cols + c] =
                v[fp4_code(q, cols, r, c)] * s[sc[(size_t)r * (cols / 16) + c / 16]] * (double)s_tensor;
}

void orc_dequant_bf16(const uint16_t* w, size_t count, double* out)
{
    for (size_t i = 0; i < count; i++) out[i] = bf16_to_double(w[i]);
}

/* ------------------------------------------------------------------ */
/* activation terms: the operand encoding of the FP4 tensor-core path   */
/* ------------------------------------------------------------------ */

/*
 * The FP4 tensor cores multiply E2M1 values with a block scale on both
 * operands, so the GPU path writes each activation row as a short sum of
 * E2M1 terms.  The pages name the weight formats only ("FreeToken
 * quantization", "Formatos compatibles, hardware y perfil de rendimiento");
 * this encoding is the library's own, and what it must match is stated
 * here, step by step, in fp32 with one rounding per operation:
 *
 *  - blocks of vs columns: vs = 32 with E8M0 scales (MXFP4 weights), vs = 16
 *    with unsigned E4M3 scales (NVFP4 weights);
 *  - NVFP4 only: the row is first multiplied by 2^p, p the integer with
 *    2^10 <= 2^p max|x| < 2^11 (p = 0 for an all-zero row), clamped to
 *    [-100, 100];
 *  - each block starts with r = x; term t = 0..T-1 takes m = max |r|, the
 *    scale s = the smallest positive value of the scale format with
 *    6 s >= m (E8M0: codes 1..254; E4M3: codes 1..0x7E, against m / 6
 *    rounded to fp32; the largest code if none qualifies), or code 127
 *    (E8M0) / 0x38 (E4M3) when m is 0; then for each element the E2M1 code
 *    nearest to r / s (ties to the code with an even mantissa bit, +0 for
 *    zero), and r <- r - e2m1(code) * s.
 *
 * codes: [T][K] one E2M1 code per byte; scales: [T][K / vs] scale codes;
 * *p_out: the row exponent.  Brute-force searches throughout.
 */
static int e2m1_nearest_code(float x)
{
    const float a = fabsf(x);
    int best = 0;
    float bd = INFINITY;
    for (int c = 0; c < 8; c++) {
        const float d = fabsf(a - (float)orc_e2m1(c));
        if (d < bd || (d == bd && (c & 1) == 0)) {
            bd = d;
            best = c;
        }
    }
    if (x < 0.0f && best != 0) best |= 8;
    return best;
}

static int term_scale_code(int wfmt, float m)
{
    if (!(m > 0.0f)) return wfmt == 1 ? 127 : 0x38;
    if (wfmt == 1) {
        for (int c = 1; c <= 254; c++)
            if (6.0 * orc_e8m0(c) >= (double)m) return c;
        return 254;
    }
    const float target = m / 6.0f;
    for (int c = 1; c <= 0x7E; c++)
        if ((float)orc_e4m3(c) >= target) return c;
    return 0x7E;
}

int orc_act_terms(const float* x, int K, int wfmt, int T, uint8_t* codes, uint8_t* scales, int* p_out)
{
    if (K <= 0 || T <= 0 || (wfmt != 1 && wfmt != 2)) return ORC_ERR_ARG;
    const int vs = wfmt == 1 ? 32 : 16;
    if (K % vs) return ORC_ERR_ARG;
    int p = 0;
    if (wfmt == 2) {
        float mx = 0.0f;
        for (int i = 0; i < K; i++) mx = fmaxf(mx, fabsf(x[i]));
        if (mx > 0.0f && mx <= 3.4e38f) {
            p = 0;
            while (ldexp((double)mx, p) >= 2048.0) p--;
            while (ldexp((double)mx, p) < 1024.0) p++;
            if (p < -100) p = -100;
            if (p > 100) p = 100;
        }
    }
    *p_out = p;
    const float sc = (float)ldexp(1.0, p);
    float r[32];
    for (int b = 0; b < K / vs; b++) {
        for (int i = 0; i < vs; i++) r[i] = wfmt == 2 ? x[b * vs + i] * sc : x[b * vs + i];
        for (int t = 0; t < T; t++) {
            float m = 0.0f;
            for (int i = 0; i < vs; i++) m = fmaxf(m, fabsf(r[i]));
            const int sc_code = term_scale_code(wfmt, m);
            const float s = m > 0.0f ? (float)(wfmt == 1 ? orc_e8m0(sc_code) : orc_e4m3(sc_code)) : 1.0f;
            scales[(size_t)t * (K / vs) + b] = (uint8_t)sc_code;
            for (int i = 0; i < vs; i++) {
                const int q = e2m1_nearest_code(r[i] / s);
                codes[(size_t)t * K + b * vs + i] = (uint8_t)q;
                const float qs = (float)orc_e2m1(q) * s;
                r[i] = r[i] - qs;
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* router: logits, top-k, renormalised softmax weights                 */
/* ------------------------------------------------------------------ */

/* One logit in the kernel's order.  32 lanes; lane l owns the 8-element
 * chunks c = l, l+32, l+64, ... of the hidden dimension and accumulates
 * acc = fmaf(x, wg, acc) over them in ascending order; the 32 partial sums
 * are then combined by an xor butterfly (offsets 16, 8, 4, 2, 1), which
 * leaves the same value in every lane. */
static float canonical_dot(const float* x, const float* w, int h)
{
    float lane[32], next[32];
    int chunks = h / 8;
    for (int l = 0; l < 32; l++) {
        float acc = 0.0f;
        for (int c = l; c < chunks; c += 32)
            for (int i = 0; i < 8; i++) acc = fmaf(x[8 * c + i], w[8 * c + i], acc);
        lane[l] = acc;
    }
    for (int off = 16; off >= 1; off >>= 1) {
        for (int l = 0; l < 32; l++) next[l] = lane[l] + lane[l ^ off];
        memcpy(lane, next, sizeof lane);
    }
    return lane[0];
}

/* a ranks above b: larger logit, ties to the lower index, NaN lowest. */
static int ranks_above(float a, int ia, float b, int ib)
{
    int na = isnan(a), nb = isnan(b);
    if (na != nb) return nb;
    if (na) return ia < ib;
    if (a != b) return a > b;
    return ia < ib;
}

/*
 * x [n][h] and wg [e][h] are the activations and the gate matrix, widened
 * exactly to float.  bias [e] may be NULL.
 * logits [n][e]: fl32(dot + bias).  idx [n][k]: the k best experts by
 * logit in descending order.  w [n][k]: exp(l_j - l_max) over the selected
 * set, normalised to sum 1 (softmax over all experts followed by
 * renormalisation over the top-k gives the same numbers).
 */
int orc_router(const float* x, const float* wg, const float* bias, int n, int h, int e, int k,
               float* logits, int32_t* idx, double* w)
{
    if (n < 0 || h <= 0 || h % 8 || e <= 0 || k <= 0 || k > e) return ORC_ERR_ARG;
    char* taken = (char*)malloc((size_t)e);
    for (int t = 0; t < n; t++) {
        float* lt = logits + (size_t)t * e;
        for (int j = 0; j < e; j++) {
            float d = canonical_dot(x + (size_t)t * h, wg + (size_t)j * h, h);
            lt[j] = bias ? d + bias[j] : d;
        }
        memset(taken, 0, (size_t)e);
        for (int r = 0; r < k; r++) {
            int best = -1;
            for (int j = 0; j < e; j++)
                if (!taken[j] && (best < 0 || ranks_above(lt[j], j, lt[best], best))) best = j;
            taken[best] = 1;
            idx[(size_t)t * k + r] = best;
        }
        double lmax = lt[idx[(size_t)t * k]], z = 0.0;
        for (int r = 0; r < k; r++) z += exp((double)lt[idx[(size_t)t * k + r]] - lmax);
        for (int r = 0; r < k; r++)
            w[(size_t)t * k + r] = exp((double)lt[idx[(size_t)t * k + r]] - lmax) / z;
    }
    free(taken);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* LRU expert-slot cache shared by all layers                          */
/* ------------------------------------------------------------------ */

enum { EV_HIT = 0, EV_MISS = 1, EV_EVICT = 2, EV_MOVE = 3 };

typedef struct {
    uint32_t call;   /* 1-based call number (the LRU clock) */
    int32_t slot;    /* slot the record refers to */
    uint16_t layer;  /* key of the record */
    uint16_t expert;
    uint8_t event;   /* EV_* */
    uint8_t pad[3];
} orc_rec;

typedef struct {
    int layers, experts, capacity;
    uint32_t clock;      /* number of lookup calls so far */
    int32_t* slot_of;    /* [layers*experts] slot or -1 */
    int32_t* key_of;     /* [capacity] layer*experts+expert or -1 (free) */
    uint64_t* stamp;     /* [capacity] clock value of the last use */
} orc_lru;

orc_lru* orc_lru_create(int layers, int experts, int capacity)
{
    if (layers <= 0 || experts <= 0 || capacity <= 0) return NULL;
    orc_lru* s = (orc_lru*)calloc(1, sizeof *s);
    s->layers = layers;
    s->experts = experts;
    s->capacity = capacity;
    s->slot_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)layers * experts);
    s->key_of = (int32_t*)malloc(sizeof(int32_t) * (size_t)capacity);
    s->stamp = (uint64_t*)calloc((size_t)capacity, sizeof(uint64_t));
    for (int i = 0; i < layers * experts; i++) s->slot_of[i] = -1;
    for (int i = 0; i < capacity; i++) s->key_of[i] = -1;
    return s;
}

void orc_lru_destroy(orc_lru* s)
{
    if (!s) return;
    free(s->slot_of);
    free(s->key_of);
    free(s->stamp);
    free(s);
}

static void put(orc_rec* out, int cap, int* n, uint32_t call, int slot, int key, int experts, int ev)
{
    if (*n < cap) {
        orc_rec* r = &out[*n];
        memset(r, 0, sizeof *r);
        r->call = call;
        r->slot = slot;
        r->layer = (uint16_t)(key / experts);
        r->expert = (uint16_t)(key % experts);
        r->event = (uint8_t)ev;
    }
    (*n)++;
}

/*
 * One lookup: layer `layer` requests the experts listed in idx[0..count).
 * R = the distinct requested experts, ascending.  |R| > capacity is an
 * error and leaves the state unchanged.  The clock advances by one.
 *  - every hit (ascending expert id): stamp <- clock, record HIT;
 *  - every miss (ascending expert id), one after the other: take the
 *    lowest-numbered free slot; if none is free, evict the resident slot
 *    with the smallest (stamp, slot) whose key is not in R (record EVICT
 *    with the evicted key); then install the key, stamp <- clock, record
 *    MISS.
 * slot_out[e] (experts entries) receives the slot of every requested
 * expert and -1 elsewhere.  Records go to out (at most cap are stored);
 * *n_out is the number produced.
 */
int orc_lru_call(orc_lru* s, int layer, const int32_t* idx, int count, int32_t* slot_out,
                 orc_rec* out, int cap, int* n_out)
{
    int E = s->experts;
    *n_out = 0;
    if (layer < 0 || layer >= s->layers) return ORC_ERR_ARG;
    char* req = (char*)calloc((size_t)E, 1);
    int nreq = 0;
    for (int i = 0; i < count; i++) {
        if (idx[i] < 0 || idx[i] >= E) { free(req); return ORC_ERR_ARG; }
        if (!req[idx[i]]) { req[idx[i]] = 1; nreq++; }
    }
    if (nreq > s->capacity) { free(req); return ORC_ERR_CAPACITY; }
    uint32_t T = ++s->clock;
    int n = 0;
    for (int e = 0; e < E; e++) {
        int key = layer * E + e;
        if (req[e] && s->slot_of[key] >= 0) {
            s->stamp[s->slot_of[key]] = T;
            put(out, cap, &n, T, s->slot_of[key], key, E, EV_HIT);
        }
    }
    for (int e = 0; e < E; e++) {
        int key = layer * E + e;
        if (!req[e] || s->slot_of[key] >= 0) continue;
        int slot = -1;
        for (int i = 0; i < s->capacity && slot < 0; i++)
            if (s->key_of[i] < 0) slot = i;
        if (slot < 0) {
            for (int i = 0; i < s->capacity; i++) {
                int k2 = s->key_of[i];
                int in_r = (k2 / E == layer) && req[k2 % E];
                if (in_r) continue;
                if (slot < 0 || s->stamp[i] < s->stamp[slot]) slot = i;
            }
            int old = s->key_of[slot];
            put(out, cap, &n, T, slot, old, E, EV_EVICT);
            s->slot_of[old] = -1;
        }
        s->key_of[slot] = key;
        s->slot_of[key] = slot;
        s->stamp[slot] = T;
        put(out, cap, &n, T, slot, key, E, EV_MISS);
    }
    if (slot_out)
        for (int e = 0; e < E; e++) slot_out[e] = req[e] ? s->slot_of[layer * E + e] : -1;
    free(req);
    *n_out = n;
    return ORC_OK;
}

/*
 * Resize to new_capacity slots.  If more keys are resident than fit, the
 * surplus is evicted in ascending (stamp, slot) order (record EVICT).  The
 * survivors are then packed into slots 0..m-1 in ascending order of their
 * old slot (record MOVE for each survivor whose slot number changes), and
 * the remaining new slots are free.  Stamps travel with their keys; the
 * clock is unchanged; records carry the current clock value.
 */
int orc_lru_resize(orc_lru* s, int new_capacity, orc_rec* out, int cap, int* n_out)
{
    int E = s->experts, C = s->capacity, n = 0;
    *n_out = 0;
    if (new_capacity <= 0) return ORC_ERR_ARG;
    int resident = 0;
    for (int i = 0; i < C; i++) resident += s->key_of[i] >= 0;
    while (resident > new_capacity) {
        int v = -1;
        for (int i = 0; i < C; i++)
            if (s->key_of[i] >= 0 && (v < 0 || s->stamp[i] < s->stamp[v])) v = i;
        put(out, cap, &n, s->clock, v, s->key_of[v], E, EV_EVICT);
        s->slot_of[s->key_of[v]] = -1;
        s->key_of[v] = -1;
        resident--;
    }
    int32_t* key2 = (int32_t*)malloc(sizeof(int32_t) * (size_t)new_capacity);
    uint64_t* st2 = (uint64_t*)calloc((size_t)new_capacity, sizeof(uint64_t));
    for (int i = 0; i < new_capacity; i++) key2[i] = -1;
    int m = 0;
    for (int i = 0; i < C; i++) {
        if (s->key_of[i] < 0) continue;
        key2[m] = s->key_of[i];
        st2[m] = s->stamp[i];
        s->slot_of[s->key_of[i]] = m;
        if (m != i) put(out, cap, &n, s->clock, m, s->key_of[i], E, EV_MOVE);
        m++;
    }
    free(s->key_of);
    free(s->stamp);
    s->key_of = key2;
    s->stamp = st2;
    s->capacity = new_capacity;
    *n_out = n;
    return ORC_OK;
}

/* Copies of the state for invariant checks. */
void orc_lru_state(const orc_lru* s, int32_t* slot_of, int32_t* key_of, uint64_t* stamp)
{
    if (slot_of) memcpy(slot_of, s->slot_of, sizeof(int32_t) * (size_t)s->layers * s->experts);
    if (key_of) memcpy(key_of, s->key_of, sizeof(int32_t) * (size_t)s->capacity);
    if (stamp) memcpy(stamp, s->stamp, sizeof(uint64_t) * (size_t)s->capacity);
}

int orc_lru_capacity(const orc_lru* s) { return s->capacity; }
uint32_t orc_lru_clock(const orc_lru* s) { return s->clock; }

/* ------------------------------------------------------------------ */
/* token -> expert permutation                                         */
/* ------------------------------------------------------------------ */

/*
 * Assignment a = t*k + j routes token t to expert idx[a].
 * counts[e] = #{a : idx[a] = e}; offsets = exclusive prefix sum (E+1
 * entries); row_of[a] = offsets[e] + #{a' < a : idx[a'] = e};
 * assign_of[row_of[a]] = a.
 */
int orc_permute(const int32_t* idx, int n, int e, int k, int32_t* offsets, int32_t* row_of,
                int32_t* assign_of)
{
    int A = n * k;
    int32_t* fill = (int32_t*)calloc((size_t)e, sizeof(int32_t));
    for (int i = 0; i <= e; i++) offsets[i] = 0;
    for (int a = 0; a < A; a++) {
        if (idx[a] < 0 || idx[a] >= e) { free(fill); return ORC_ERR_ARG; }
        offsets[idx[a] + 1]++;
    }
    for (int i = 0; i < e; i++) offsets[i + 1] += offsets[i];
    for (int a = 0; a < A; a++) {
        int r = offsets[idx[a]] + fill[idx[a]]++;
        row_of[a] = r;
        assign_of[r] = a;
    }
    free(fill);
    return ORC_OK;
}

/* ------------------------------------------------------------------ */
/* expert FFN (SwiGLU) and combine                                     */
/* ------------------------------------------------------------------ */

/*
 * One token through one expert.  w13 [2F][H] (rows 0..F-1 gate W1, rows
 * F..2F-1 up W3), w2 [H][F], all real-valued; x [H].
 * g = W1 x, u = W3 x, h = silu(g) * u with silu(z) = z / (1 + exp(-z)),
 * y = W2 h.  fp64 throughout.
 */
void orc_expert_ffn(const double* w13, const double* w2, int h, int f, const double* x, double* y)
{
    double* hv = (double*)malloc(sizeof(double) * (size_t)f);
    for (int i = 0; i < f; i++) {
        double g = 0.0, u = 0.0;
        const double* r1 = w13 + (size_t)i * h;
        const double* r3 = w13 + (size_t)(f + i) * h;
        for (int c = 0; c < h; c++) {
            g += r1[c] * x[c];
            u += r3[c] * x[c];
        }
        hv[i] = g / (1.0 + exp(-g)) * u;
    }
    for (int o = 0; o < h; o++) {
        double acc = 0.0;
        const double* r2 = w2 + (size_t)o * f;
        for (int i = 0; i < f; i++) acc += r2[i] * hv[i];
        y[o] = acc;
    }
    free(hv);
}

/* out[t] = sum over j = 0..k-1, in order, of w[t][j] * y[t*k+j]. */
void orc_combine(const double* y, const double* w, int n, int k, int h, double* out)
{
    for (int t = 0; t < n; t++)
        for (int c = 0; c < h; c++) {
            double acc = 0.0;
            for (int j = 0; j < k; j++)
                acc += w[(size_t)t * k + j] * y[((size_t)t * k + j) * h + c];
            out[(size_t)t * h + c] = acc;
        }
}
