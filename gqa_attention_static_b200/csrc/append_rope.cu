// append_rope.cu -- RoPE on the new query/key rows and the delta write into
// the static cache.
//
// "ARK-ASR-3B -- INT8 ONNX" model card, section Shapes: the decoder returns
// key_delta_i / value_delta_i rows for the positions written by this call, and
// the host copies them into cache_{key,value}_i at cache_position.  Here that
// copy is a device-side scatter fused with the rotary embedding of the new
// rows (Qwen2 rotate-half form: SGLang-Omni cookbook "ARK-ASR-3B",
// introduction).
//
// Rounding: table entries are fp32, inputs bf16, so every product is exact in
// double; each output x[i]*c - x[i+64]*s (or x[i+64]*c + x[i]*s) is one double
// subtraction/addition rounded once to bf16 with cvt.rn.bf16.f64.  The result
// is therefore bit-reproducible.
//
// fp8 cache variant (ark_attn_append_rope_fp8): the caches hold OCP E4M3
// codes with one fp32 scale per (layer, KV head) for K and one for V, stored
// head-major (a cache format the pages do not have; they quantise weights
// only).  The rotated key
// is divided by its scale in double (not rounded to bf16 first), rounded to
// fp32 and converted to e4m3 with cvt.rn.satfinite; values likewise.  q is
// rotated to bf16 exactly as above.
//
// Work: one CTA per (request, layer) and group of rows (one row for a decode
// step, 8 consecutive rows of a prompt, so that a long padded prompt batch
// does not launch a CTA per padded row).  A row's items are (Hq + Hkv) heads
// x 16 groups of 4 rotary pairs plus Hkv x 16 16-byte pieces of the V copy;
// the CTA's (row, item) pairs share one index space over its threads (one
// item per thread for a decode row).  The op is small next to the attention; it exists so the caller
// never crosses to the host between the projection and the attention.
#include "common.cuh"

namespace ark {

struct AppendLayer {
    uint16_t* q;
    const uint16_t* k_new;
    const uint16_t* v_new;
    void* cache_k;           // bf16 or fp8 codes
    void* cache_v;
    const float* k_scale;    // fp8 only: [Hkv]
    const float* v_scale;
};

struct AppendParams {
    const int32_t* pos0;
    const int32_t* n_new;
    const float2* table;  // [T][64] {cos, sin}
    uint32_t* status;
    int B, S, T, Hq, Hkv;
    int rotate_q;         // 0: K/V rows only (q is rotated where it is read, by the prefill)
    int rows_per_cta;     // consecutive rows t of one (request, layer) per CTA
    AppendLayer layer[ARK_MAX_LAYERS];
};

// Byte offset of (request b, KV head g, position pos) in an fp8 cache, which
// is head-major [B][Hkv][T][128]: one head's positions are consecutive
// 128-byte rows, so a tile of positions is one contiguous block.
__device__ __forceinline__ size_t fp8_row_offset(int b, int g, int pos, int T, int Hkv) {
    return ((static_cast<size_t>(b) * Hkv + g) * T + pos) * kHeadDim;
}

template <bool Fp8>
__global__ void __launch_bounds__(512) append_rope_kernel(const __grid_constant__ AppendParams p) {
    // a kernel launched behind this one with programmatic stream serialisation
    // (the decode) may start its own prologue now; it waits for this grid's
    // completion (griddepcontrol.wait) before it reads q or the cache
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int b = blockIdx.y;
    const AppendLayer& L = p.layer[blockIdx.z];

    int nn = __ldg(p.n_new + b);
    if (nn < 0 || nn > p.S) {
        if (threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.z == 0) report(p.status, ARK_DEV_BAD_KVLEN);
        nn = nn < 0 ? 0 : p.S;
    }
    const int p0 = __ldg(p.pos0 + b);
    const int t_first = static_cast<int>(blockIdx.x) * p.rows_per_cta;
    const int nrows = min(nn, t_first + p.rows_per_cta) - t_first;
    const int qh = p.rotate_q ? p.Hq : 0;    // query heads this call rotates
    const int nrot = (qh + p.Hkv) * 16;      // items of 4 rotary pairs per row
    const int ncopy = p.Hkv * 16;            // 16-byte pieces of V rows per row
    const int nitems = nrot + ncopy;
    // (row, item) pairs of the CTA's rows in one index space, so that every
    // thread has at most a couple of items and their loads are in flight together
    for (int idx = threadIdx.x; idx < nrows * nitems; idx += blockDim.x) {
        const int t = t_first + idx / nitems;
        const int it = idx - (t - t_first) * nitems;
        const int pos = p0 + t;
        if (pos < 0 || pos >= p.T) {
            if (it == 0 && blockIdx.z == 0) report(p.status, ARK_DEV_BAD_POS);
            continue;
        }
        const float4* trow = reinterpret_cast<const float4*>(p.table + static_cast<size_t>(pos) * 64);
        {
            if (it < nrot) {
                const int head = it >> 4;
                const int pg = it & 15;           // pairs 4pg .. 4pg+3
                const uint16_t* src;
                uint16_t* dst = nullptr;
                uint8_t* dst8 = nullptr;
                double kscale = 1.0;
                if (head < qh) {
                    uint16_t* row = L.q + ((static_cast<size_t>(b) * p.S + t) * p.Hq + head) * kHeadDim;
                    src = row;
                    dst = row;
                } else {
                    const int g = head - qh;
                    src = L.k_new + ((static_cast<size_t>(b) * p.S + t) * p.Hkv + g) * kHeadDim;
                    if (Fp8) {
                        dst8 = static_cast<uint8_t*>(L.cache_k) + fp8_row_offset(b, g, pos, p.T, p.Hkv);
                        kscale = static_cast<double>(__ldg(L.k_scale + g));
                    } else {
                        dst = static_cast<uint16_t*>(L.cache_k) + ((static_cast<size_t>(b) * p.T + pos) * p.Hkv + g) * kHeadDim;
                    }
                }
                const uint2 lo = *reinterpret_cast<const uint2*>(src + 4 * pg);
                const uint2 hi = *reinterpret_cast<const uint2*>(src + 64 + 4 * pg);
                const float4 cs01 = __ldg(trow + 2 * pg);      // c0 s0 c1 s1
                const float4 cs23 = __ldg(trow + 2 * pg + 1);  // c2 s2 c3 s3
                const uint16_t xl[4] = {static_cast<uint16_t>(lo.x & 0xffff), static_cast<uint16_t>(lo.x >> 16),
                                        static_cast<uint16_t>(lo.y & 0xffff), static_cast<uint16_t>(lo.y >> 16)};
                const uint16_t xh[4] = {static_cast<uint16_t>(hi.x & 0xffff), static_cast<uint16_t>(hi.x >> 16),
                                        static_cast<uint16_t>(hi.y & 0xffff), static_cast<uint16_t>(hi.y >> 16)};
                const float cc[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
                const float ss[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
                if (Fp8 && dst8) {
                    // the key for the fp8 cache is quantised from the unrounded rotation, in double
                    double dl[4], dh[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const double a = bf16_bits_to_f64(xl[i]);
                        const double h = bf16_bits_to_f64(xh[i]);
                        const double c = static_cast<double>(cc[i]);
                        const double s = static_cast<double>(ss[i]);
                        // both products are exact in double, so contraction cannot change the result
                        dl[i] = a * c - h * s;
                        dh[i] = h * c + a * s;
                    }
                    // the key into the fp8 cache: e4m3(fp32(y / scale)), two codes per conversion
                    uint32_t cl = 0, ch = 0;
#pragma unroll
                    for (int i = 0; i < 4; i += 2) {
                        cl |= static_cast<uint32_t>(f32x2_to_e4m3x2(__double2float_rn(dl[i] / kscale),
                                                                    __double2float_rn(dl[i + 1] / kscale))) << (8 * i);
                        ch |= static_cast<uint32_t>(f32x2_to_e4m3x2(__double2float_rn(dh[i] / kscale),
                                                                    __double2float_rn(dh[i + 1] / kscale))) << (8 * i);
                    }
                    *reinterpret_cast<uint32_t*>(dst8 + 4 * pg) = cl;
                    *reinterpret_cast<uint32_t*>(dst8 + 64 + 4 * pg) = ch;
                    continue;
                }
                uint16_t yl[4], yh[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const double a = bf16_bits_to_f64(xl[i]);
                    const double h = bf16_bits_to_f64(xh[i]);
                    const double c = static_cast<double>(cc[i]);
                    const double s = static_cast<double>(ss[i]);
                    // both products are exact in double, so contraction cannot change the result
                    yl[i] = f64_to_bf16_rn(a * c - h * s);
                    yh[i] = f64_to_bf16_rn(h * c + a * s);
                }
                uint2 ol, oh;
                ol.x = static_cast<uint32_t>(yl[0]) | (static_cast<uint32_t>(yl[1]) << 16);
                ol.y = static_cast<uint32_t>(yl[2]) | (static_cast<uint32_t>(yl[3]) << 16);
                oh.x = static_cast<uint32_t>(yh[0]) | (static_cast<uint32_t>(yh[1]) << 16);
                oh.y = static_cast<uint32_t>(yh[2]) | (static_cast<uint32_t>(yh[3]) << 16);
                *reinterpret_cast<uint2*>(dst + 4 * pg) = ol;
                *reinterpret_cast<uint2*>(dst + 64 + 4 * pg) = oh;
            } else {
                const int c = it - nrot;
                const int g = c >> 4;
                const int piece = c & 15;
                const uint4* src = reinterpret_cast<const uint4*>(
                    L.v_new + ((static_cast<size_t>(b) * p.S + t) * p.Hkv + g) * kHeadDim);
                if (Fp8) {
                    // 8 values -> 8 codes: e4m3(fp32(v / scale))
                    const double vscale = static_cast<double>(__ldg(L.v_scale + g));
                    const uint4 x = src[piece];
                    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
                    uint32_t out[2] = {0, 0};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float f0 = __double2float_rn(bf16_bits_to_f64(static_cast<uint16_t>(w[i] & 0xffff)) / vscale);
                        const float f1 = __double2float_rn(bf16_bits_to_f64(static_cast<uint16_t>(w[i] >> 16)) / vscale);
                        out[i >> 1] |= static_cast<uint32_t>(f32x2_to_e4m3x2(f0, f1)) << (16 * (i & 1));
                    }
                    *reinterpret_cast<uint2*>(static_cast<uint8_t*>(L.cache_v) + fp8_row_offset(b, g, pos, p.T, p.Hkv) +
                                              8 * piece) = make_uint2(out[0], out[1]);
                } else {
                    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(L.cache_v) +
                                                          ((static_cast<size_t>(b) * p.T + pos) * p.Hkv + g) * kHeadDim);
                    dst[piece] = src[piece];
                }
            }
        }
    }
}

}  // namespace ark

using namespace ark;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

ark_status check_common(int B, int S, int T, int Hq, int Hkv, int D) {
    if (B <= 0 || S <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return ARK_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ARK_ERR_INVALID_ARG;
    if (T > ARK_MAX_T) return ARK_ERR_UNSUPPORTED;
    if (D != kHeadDim || Hq / Hkv != kGroup) return ARK_ERR_UNSUPPORTED;
    if (B > 65535 || S > 2147483647 / 2) return ARK_ERR_UNSUPPORTED;
    return ARK_OK;
}

ark_status launch_append(AppendParams& prm, int L, bool fp8, cudaStream_t stream) {
    // K/V rows only, of a long prompt: several rows per CTA, so that the grid
    // is not a CTA per (mostly padded) row; with the query rows each row is
    // enough work for its own CTA
    prm.rows_per_cta = (prm.S >= 64 && !prm.rotate_q) ? 8 : 1;
    dim3 grid((prm.S + prm.rows_per_cta - 1) / prm.rows_per_cta, prm.B, L);
    // one thread per item of a row with the query heads ((Hq + 2 Hkv) x 16 = 320 for the
    // decoder's heads), two per item of the eight K/V-only rows of a CTA otherwise
    const int items = ((prm.rotate_q ? prm.Hq : 0) + 2 * prm.Hkv) * 16 * prm.rows_per_cta;
    int threads = items < 512 ? ((items + 31) / 32) * 32 : 256;
    if (threads > 512) threads = 512;
    if (fp8)
        append_rope_kernel<true><<<grid, threads, 0, stream>>>(prm);
    else
        append_rope_kernel<false><<<grid, threads, 0, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

}  // namespace

extern "C" ark_status ark_attn_append_rope(void* q, const void* k_new, const void* v_new,
                                           void* cache_k, void* cache_v,
                                           const int32_t* pos0, const int32_t* n_new,
                                           int B, int S, int T, int Hq, int Hkv, int D,
                                           const float* d_table, uint32_t* d_status,
                                           cudaStream_t stream) {
    if (!q || !k_new || !v_new || !cache_k || !cache_v || !pos0 || !n_new || !d_table)
        return ARK_ERR_INVALID_ARG;
    ark_status st = check_common(B, S, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (S > 65535) return ARK_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(cache_k) ||
        !aligned16(cache_v) || !aligned16(d_table))
        return ARK_ERR_INVALID_ARG;
    AppendParams prm{};
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.table = reinterpret_cast<const float2*>(d_table);
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    prm.rotate_q = 1;
    prm.layer[0] = AppendLayer{static_cast<uint16_t*>(q), static_cast<const uint16_t*>(k_new),
                               static_cast<const uint16_t*>(v_new), cache_k, cache_v, nullptr, nullptr};
    return launch_append(prm, 1, false, stream);
}

extern "C" ark_status ark_attn_append_rope_layers(int L, void* const* q, const void* const* k_new,
                                                  const void* const* v_new, void* const* cache_k,
                                                  void* const* cache_v, const int32_t* pos0,
                                                  const int32_t* n_new, int B, int S, int T, int Hq, int Hkv,
                                                  int D, const float* d_table, uint32_t* d_status,
                                                  cudaStream_t stream) {
    if (!q || !k_new || !v_new || !cache_k || !cache_v || !pos0 || !n_new || !d_table)
        return ARK_ERR_INVALID_ARG;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    ark_status st = check_common(B, S, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (S > 65535) return ARK_ERR_UNSUPPORTED;
    if (!aligned16(d_table)) return ARK_ERR_INVALID_ARG;
    AppendParams prm{};
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.table = reinterpret_cast<const float2*>(d_table);
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    prm.rotate_q = 1;
    for (int l = 0; l < L; ++l) {
        if (!q[l] || !k_new[l] || !v_new[l] || !cache_k[l] || !cache_v[l]) return ARK_ERR_INVALID_ARG;
        if (!aligned16(q[l]) || !aligned16(k_new[l]) || !aligned16(v_new[l]) || !aligned16(cache_k[l]) ||
            !aligned16(cache_v[l]))
            return ARK_ERR_INVALID_ARG;
        prm.layer[l] = AppendLayer{static_cast<uint16_t*>(q[l]), static_cast<const uint16_t*>(k_new[l]),
                                   static_cast<const uint16_t*>(v_new[l]), cache_k[l], cache_v[l], nullptr, nullptr};
    }
    return launch_append(prm, L, false, stream);
}

extern "C" ark_status ark_attn_append_rope_fp8_layers(int L, void* const* q, const void* const* k_new,
                                                      const void* const* v_new, void* const* cache_k,
                                                      void* const* cache_v, const float* const* k_scale,
                                                      const float* const* v_scale, const int32_t* pos0,
                                                      const int32_t* n_new, int B, int S, int T, int Hq, int Hkv,
                                                      int D, const float* d_table, uint32_t* d_status,
                                                      cudaStream_t stream) {
    if (!q || !k_new || !v_new || !cache_k || !cache_v || !k_scale || !v_scale || !pos0 || !n_new || !d_table)
        return ARK_ERR_INVALID_ARG;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    ark_status st = check_common(B, S, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (S > 65535) return ARK_ERR_UNSUPPORTED;
    if (!aligned16(d_table)) return ARK_ERR_INVALID_ARG;
    AppendParams prm{};
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.table = reinterpret_cast<const float2*>(d_table);
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    prm.rotate_q = 1;
    for (int l = 0; l < L; ++l) {
        if (!q[l] || !k_new[l] || !v_new[l] || !cache_k[l] || !cache_v[l] || !k_scale[l] || !v_scale[l])
            return ARK_ERR_INVALID_ARG;
        if (!aligned16(q[l]) || !aligned16(k_new[l]) || !aligned16(v_new[l]) || !aligned16(cache_k[l]) ||
            !aligned16(cache_v[l]) || !aligned4(k_scale[l]) || !aligned4(v_scale[l]))
            return ARK_ERR_INVALID_ARG;
        prm.layer[l] = AppendLayer{static_cast<uint16_t*>(q[l]), static_cast<const uint16_t*>(k_new[l]),
                                   static_cast<const uint16_t*>(v_new[l]), cache_k[l], cache_v[l], k_scale[l],
                                   v_scale[l]};
    }
    return launch_append(prm, L, true, stream);
}

extern "C" ark_status ark_attn_append_rope_fp8(void* q, const void* k_new, const void* v_new, void* cache_k,
                                               void* cache_v, const float* k_scale, const float* v_scale,
                                               const int32_t* pos0, const int32_t* n_new, int B, int S, int T,
                                               int Hq, int Hkv, int D, const float* d_table, uint32_t* d_status,
                                               cudaStream_t stream) {
    const void* kn = k_new;
    const void* vn = v_new;
    return ark_attn_append_rope_fp8_layers(1, &q, &kn, &vn, &cache_k, &cache_v, &k_scale, &v_scale, pos0, n_new,
                                           B, S, T, Hq, Hkv, D, d_table, d_status, stream);
}

extern "C" ark_status ark_attn_append_rope_kv_layers(int L, const void* const* k_new, const void* const* v_new,
                                                     void* const* cache_k, void* const* cache_v, const int32_t* pos0,
                                                     const int32_t* n_new, int B, int S, int T, int Hq, int Hkv,
                                                     int D, const float* d_table, uint32_t* d_status,
                                                     cudaStream_t stream) {
    if (!k_new || !v_new || !cache_k || !cache_v || !pos0 || !n_new || !d_table) return ARK_ERR_INVALID_ARG;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    ark_status st = check_common(B, S, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (S > 65535) return ARK_ERR_UNSUPPORTED;
    if (!aligned16(d_table)) return ARK_ERR_INVALID_ARG;
    AppendParams prm{};
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.table = reinterpret_cast<const float2*>(d_table);
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    prm.rotate_q = 0;
    for (int l = 0; l < L; ++l) {
        if (!k_new[l] || !v_new[l] || !cache_k[l] || !cache_v[l]) return ARK_ERR_INVALID_ARG;
        if (!aligned16(k_new[l]) || !aligned16(v_new[l]) || !aligned16(cache_k[l]) || !aligned16(cache_v[l]))
            return ARK_ERR_INVALID_ARG;
        prm.layer[l] = AppendLayer{nullptr, static_cast<const uint16_t*>(k_new[l]),
                                   static_cast<const uint16_t*>(v_new[l]), cache_k[l], cache_v[l], nullptr, nullptr};
    }
    return launch_append(prm, L, false, stream);
}

extern "C" ark_status ark_attn_append_rope_kv(const void* k_new, const void* v_new, void* cache_k, void* cache_v,
                                              const int32_t* pos0, const int32_t* n_new, int B, int S, int T,
                                              int Hq, int Hkv, int D, const float* d_table, uint32_t* d_status,
                                              cudaStream_t stream) {
    return ark_attn_append_rope_kv_layers(1, &k_new, &v_new, &cache_k, &cache_v, pos0, n_new, B, S, T, Hq, Hkv, D,
                                          d_table, d_status, stream);
}
