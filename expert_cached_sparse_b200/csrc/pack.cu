// Host-side packing of one expert from the canonical layout into the slot
// blob the kernels stream.  The pages describe a runtime weight format that
// keeps the expert banks already laid out as the runtime uses them, so
// start-up needs no tensor discovery or repacking ("FreeToken linux",
// section "Prepara los pesos del modelo"; "FreeToken 290b model", section
// "Identifica el modelo y el formato de expertos").  This is that layout for
// this library; one fill is one contiguous copy of it.  The layout is
// described in common.cuh (BlobLayout).
#include <math.h>
#include <string.h>

#include "common.cuh"

namespace {

// BF16: canonical row of packed W13 row p (tile rows 0..7 gate f, 8..15 up f)
inline int w13_canon_row(int p, int F)
{
    int rt = p / 16, r = p % 16;
    int f = 8 * rt + (r & 7);
    return r < 8 ? f : F + f;
}

// FP4: canonical row of row r of W13 row block G (per 32 rows: 16 gate rows,
// then the 16 matching up rows)
inline int w13_canon_row(int G, int r, int F)
{
    const int q = r / 32, i = r % 32;
    const int f = 64 * G + 16 * q + (i % 16);
    return i < 16 ? f : F + f;
}

// FP4 matrix [R][K] (codes two per byte, scales [R][K / vs]) -> chunk images
// (common.cuh): per 128-row block and 256-column chunk, the rows' code bytes
// in the 128-byte swizzle, then the unsigned block scales in tensor-memory
// copy order.  NVFP4 blocks with a negative scale get their codes negated.
void pack_fp4_matrix(const uint8_t* q, const uint8_t* sc, int R, int K, bool w13, int F, int wfmt, uint8_t* out)
{
    const bool nv = wfmt == MOE_W_NVFP4;
    const int vs = nv ? 16 : 32, KC = K / 256, spc = 256 / vs;   // scales per row per chunk
    const size_t cb = (size_t)moe::fp4_chunk_bytes(wfmt);
    for (int G = 0; G < R / 128; G++)
        for (int c = 0; c < KC; c++) {
            uint8_t* img = out + ((size_t)G * KC + c) * cb;
            for (int r = 0; r < 128; r++) {
                const int cr = w13 ? w13_canon_row(G, r, F) : 128 * G + r;
                const uint8_t* src = q + (size_t)cr * (K / 2) + 128 * c;
                const uint8_t* srow = sc + (size_t)cr * (K / vs) + (size_t)spc * c;
                for (int b = 0; b < 128; b++) {
                    uint8_t v = src[b];
                    if (nv && (srow[b / 8] & 0x80)) v ^= 0x88;   // 8 bytes per 16-column block
                    img[1024 * (r / 8) + 128 * (r % 8) + 16 * ((b / 16) ^ (r % 8)) + (b % 16)] = v;
                }
                for (int si = 0; si < spc; si++)
                    img[16384 + 512 * (si / 4) + 16 * (r % 32) + 4 * (r / 32) + (si % 4)] =
                        nv ? (uint8_t)(srow[si] & 0x7F) : srow[si];
            }
        }
}

// BF16 tile: for k16 step j, lane L = 4g+t holds 16 bytes
// {a0, a2, a1, a3}: rows g / g+8, column pairs (16j+2t, +1) and (16j+8+2t, +1).
void pack_bf16_matrix(const uint16_t* w, int R, int K, bool w13, int F, uint8_t* out)
{
    const int KT = K / 64;
    for (int rt = 0; rt < R / 16; rt++)
        for (int kt = 0; kt < KT; kt++) {
            uint8_t* tile = out + moe::tile_index(rt, kt, R / 16, KT) * 2048;
            for (int j = 0; j < 4; j++)
                for (int L = 0; L < 32; L++) {
                    int g = L >> 2, t = L & 3;
                    for (int half = 0; half < 2; half++) {
                        int p = 16 * rt + g + 8 * half;
                        int cr = w13 ? w13_canon_row(p, F) : p;
                        const uint16_t* src = w + (size_t)cr * K + 64 * kt + 16 * j + 2 * t;
                        uint8_t* dst = tile + 512 * j + 16 * L;
                        memcpy(dst + 8 * half, src, 4);          // a0 / a1
                        memcpy(dst + 8 * half + 4, src + 8, 4);  // a2 / a3
                    }
                }
        }
}

// E8M0 code 255 is NaN; every other code is a finite power of two.
bool mx_codes_ok(const uint8_t* sc, size_t n)
{
    for (size_t i = 0; i < n; i++)
        if (sc[i] == 255) return false;
    return true;
}

bool nv_codes_ok(const uint8_t* sc, size_t n)
{
    for (size_t i = 0; i < n; i++)
        if ((sc[i] & 0x7F) == 0x7F) return false;   // S.1111.111 is NaN
    return true;
}

}  // namespace

extern "C" size_t moe_slot_bytes(const moe_shape* shape)
{
    if (!moe::shape_ok(shape)) return 0;
    return moe::blob_layout(shape).bytes;
}

extern "C" int moe_pack_expert(const moe_shape* s, const void* h_w13, const uint8_t* h_w13_scales,
                               const void* h_w2, const uint8_t* h_w2_scales, const float* h_tensor_scales,
                               void* h_blob_out)
{
    if (!moe::shape_ok(s) || !h_w13 || !h_w2 || !h_blob_out) return MOE_ERR_INVALID_ARG;
    const int H = s->hidden, F = s->ffn;
    moe::BlobLayout bl = moe::blob_layout(s);
    uint8_t* out = static_cast<uint8_t*>(h_blob_out);
    memset(out, 0, bl.bytes);
    if (s->wfmt == MOE_W_BF16) {
        pack_bf16_matrix(static_cast<const uint16_t*>(h_w13), 2 * F, H, true, F, out + bl.w13);
        pack_bf16_matrix(static_cast<const uint16_t*>(h_w2), H, F, false, F, out + bl.w2);
        return MOE_OK;
    }
    if (!h_w13_scales || !h_w2_scales) return MOE_ERR_INVALID_ARG;
    const bool mx = s->wfmt == MOE_W_MXFP4;
    const size_t per = mx ? 32 : 16;
    const size_t n13 = (size_t)2 * F * H / per, n2 = (size_t)H * F / per;
    if (mx) {
        if (!mx_codes_ok(h_w13_scales, n13) || !mx_codes_ok(h_w2_scales, n2)) return MOE_ERR_UNSUPPORTED;
    } else {
        if (!h_tensor_scales) return MOE_ERR_INVALID_ARG;
        if (!nv_codes_ok(h_w13_scales, n13) || !nv_codes_ok(h_w2_scales, n2)) return MOE_ERR_UNSUPPORTED;
        for (int i = 0; i < 2; i++)
            if (!isfinite(h_tensor_scales[i])) return MOE_ERR_UNSUPPORTED;
    }
    pack_fp4_matrix(static_cast<const uint8_t*>(h_w13), h_w13_scales, 2 * F, H, true, F, s->wfmt, out + bl.w13);
    pack_fp4_matrix(static_cast<const uint8_t*>(h_w2), h_w2_scales, H, F, false, F, s->wfmt, out + bl.w2);
    if (!mx) memcpy(out + bl.ts, h_tensor_scales, 2 * sizeof(float));
    return MOE_OK;
}
