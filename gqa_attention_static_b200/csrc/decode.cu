// decode.cu -- split-KV single-token GQA decode over a ragged batch, and the
// log-sum-exp merge of its partial results.
//
// The attention is the decoder's, over the static cache of the "ARK-ASR-3B --
// INT8 ONNX" model card (section Shapes): 16 query heads, 2 KV heads, head dim
// 128, cache [B, T, 2, 128] sequence-major.  The static graph the card
// describes attends over all T = max_total_len positions on every token;
// here the length-aware mode reads only the kv_len[b] valid rows, and the
// masked-static mode reproduces the card's behaviour (read all T rows, score
// the invalid ones -inf) so the two can be timed side by side.
//
// Design (B200):
//   - One CTA per (split, KV head g, request b, layer).  The 8 query heads of
//     group g are served from a single read of each K/V row.
//   - Each of the 4 warps owns a private 2-stage ring of 16-row K/V tiles in
//     shared memory, filled by the TMA engine with 1-D bulk copies (one 256 B
//     row per copy, completion counted on an mbarrier).  Rows are padded to
//     272 B so that ldmatrix reads are bank-conflict free.
//   - Scores are computed transposed, S^T[16 pos x 8 heads] = K_tile * Q^T,
//     with m16n8k16 bf16 tensor-core MMAs: positions fill M = 16 and the 8
//     heads of the group fill N = 8 exactly, so no MMA lane is wasted.  P^T is
//     moved from the accumulator layout to the B-operand layout with two
//     movmatrix transposes, and O^T[dims x heads] += V^T * P^T uses
//     ldmatrix.trans on the same V tile.
//   - fp32 online softmax in the log2 domain; per-head max across the 16
//     positions by warp shuffles.  The four warps merge in shared memory;
//     with one split the CTA writes o/lse directly, otherwise fp32 partials.
//
// Why tensor cores: per (position, KV head) the kernel reads 512 B and does
// 2 x 8 x 128 multiply-adds, 4 FMA per byte.  At B200 HBM rates that needs
// most of the fp32 FMA pipe; on the tensor pipe it is a few percent.
#include "common.cuh"

namespace ark {

constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kRowPitch = 272;                      // bytes per smem row (256 + 16 pad)
constexpr int kTileRows = 16;
constexpr int kTileBytes = kTileRows * kRowPitch;   // one 16-row K or V tile
constexpr int kStageBytes = 2 * kTileBytes;         // K tile + V tile
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kMergeBytes = kWarps * kGroup * kHeadDim * 4 + kWarps * kGroup * 2 * 4;
static_assert(kMergeBytes <= kRingBytes, "merge area aliases the rings");
constexpr int kDecodeSmem = kRingBytes + kWarps * kStages * 8 + 16;

struct DecodeLayer {
    const uint16_t* q;
    const uint16_t* k;
    const uint16_t* v;
    uint16_t* o;
    float* lse;
    float* o_part;
    float* lse_part;
};

struct DecodeParams {
    const int32_t* kv_len;
    uint32_t* status;
    int B, T, Hq, Hkv;
    int nsplit, chunk;
    int masked;
    float scale_log2;
    DecodeLayer layer[ARK_MAX_LAYERS];
};

struct CombineLayer {
    const float* o_part;
    const float* lse_part;
    uint16_t* o;
    float* lse;
};

struct CombineParams {
    int B, Hq, nsplit;
    CombineLayer layer[ARK_MAX_LAYERS];
};

// Issue the bulk copies of one 16-row tile (rows r0 .. r0+nrows-1 of KV head
// g of request b) into a stage; V rows past nrows are zeroed so that their
// zero softmax weight cannot meet a NaN.
__device__ __forceinline__ void issue_tile(uint8_t* stage, uint64_t* bar, const uint16_t* kbase,
                                           const uint16_t* vbase, int row_stride, int r0, int nrows,
                                           int lane) {
    if (lane == 0) mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nrows) * 2u * 256u);
    __syncwarp();
    fence_proxy_async_smem();
    if (lane < kTileRows) {
        if (lane < nrows)
            bulk_g2s(stage + lane * kRowPitch, kbase + static_cast<size_t>(r0 + lane) * row_stride, 256, bar);
    } else {
        const int r = lane - kTileRows;
        if (r < nrows) {
            bulk_g2s(stage + kTileBytes + r * kRowPitch, vbase + static_cast<size_t>(r0 + r) * row_stride,
                     256, bar);
        } else {
            uint4* z = reinterpret_cast<uint4*>(stage + kTileBytes + r * kRowPitch);
#pragma unroll
            for (int i = 0; i < 16; ++i) z[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

__global__ void __launch_bounds__(kWarps * 32) decode_split_kernel(const __grid_constant__ DecodeParams p) {
    extern __shared__ __align__(128) uint8_t smem[];
    const int split = blockIdx.x;
    const int g = blockIdx.y;
    const int b = blockIdx.z % p.B;
    const int l = blockIdx.z / p.B;
    const DecodeLayer& L = p.layer[l];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2;
    const int tig = lane & 3;

    int kvl = __ldg(p.kv_len + b);
    if (kvl < 0 || kvl > p.T) {
        if (threadIdx.x == 0 && split == 0 && g == 0 && l == 0) report(p.status, ARK_DEV_BAD_KVLEN);
        kvl = kvl < 0 ? 0 : p.T;
    }
    const int hi = p.masked ? p.T : kvl;          // rows read
    const int j_begin = split * p.chunk;
    const int j_end = min(j_begin + p.chunk, hi);
    const int lim = min(kvl, j_end);                // rows scored
    const int head0 = g * kGroup;

    if (j_begin >= j_end) {
        // no rows in this chunk: an empty partial (or, unsplit, o = 0 / lse = -inf)
        if (threadIdx.x < kGroup) {
            const int h = head0 + threadIdx.x;
            if (p.nsplit == 1) {
                L.lse[static_cast<size_t>(b) * p.Hq + h] = -INFINITY;
            } else {
                L.lse_part[(static_cast<size_t>(b) * p.Hq + h) * p.nsplit + split] = -INFINITY;
            }
        }
        if (p.nsplit == 1) {
            // o = 0 for the 8 heads: 8 x 128 bf16 = 128 x 16 B
            uint4* o4 = reinterpret_cast<uint4*>(L.o + (static_cast<size_t>(b) * p.Hq + head0) * kHeadDim);
            o4[threadIdx.x] = make_uint4(0, 0, 0, 0);
        }
        return;
    }

    uint8_t* ring = smem + warp * (kStages * kStageBytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRingBytes) + warp * kStages;
    int& s_failed = *reinterpret_cast<int*>(smem + kRingBytes + kWarps * kStages * 8);
    if (threadIdx.x == 0) s_failed = 0;
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    fence_proxy_async_smem();
    __syncthreads();

    const int row_stride = p.Hkv * kHeadDim;
    const uint16_t* kbase = L.k + static_cast<size_t>(b) * p.T * row_stride + g * kHeadDim;
    const uint16_t* vbase = L.v + static_cast<size_t>(b) * p.T * row_stride + g * kHeadDim;

    const int ntiles = (j_end - j_begin + kTileRows - 1) / kTileRows;
    const int my_tiles = ntiles > warp ? (ntiles - warp + kWarps - 1) / kWarps : 0;

    // prologue: fill the ring
    for (int s = 0; s < kStages && s < my_tiles; ++s) {
        const int r0 = j_begin + (warp + s * kWarps) * kTileRows;
        issue_tile(ring + s * kStageBytes, &bars[s], kbase, vbase, row_stride, r0,
                   min(kTileRows, j_end - r0), lane);
    }

    // Q of the 8 heads as B fragments: b0 = Q[head gid][16kk + 2tig .. +1], b1 = same + 8
    uint32_t qf[8][2];
    {
        const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
            L.q + (static_cast<size_t>(b) * p.Hq + head0 + gid) * kHeadDim);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            qf[kk][0] = __ldg(qrow + kk * 8 + tig);
            qf[kk][1] = __ldg(qrow + kk * 8 + 4 + tig);
        }
    }

    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY;   // running max of heads 2tig, 2tig+1 (log2 domain)
    float l0 = 0.f, l1 = 0.f;               // this lane's share of the running sums

    // ldmatrix lane roles
    const int lr = lane & 7;
    const int lm = lane >> 3;
    const uint32_t ring_u32 = smem_u32(ring);
    // K (A operand, non-transposed): matrix lm -> rows 8*(lm&1), cols 8*(lm>>1)
    const uint32_t k_off = (lr + 8 * (lm & 1)) * kRowPitch + 16 * (lm >> 1);
    // V (A operand of V^T, transposed load): matrix lm -> rows 8*(lm>>1), cols 8*(lm&1)
    const uint32_t v_off = kTileBytes + (lr + 8 * (lm >> 1)) * kRowPitch + 16 * (lm & 1);

    bool failed = false;
    int failed_at = 0;
    for (int it = 0; it < my_tiles; ++it) {
        const int s = it % kStages;
        const uint32_t parity = (it / kStages) & 1;
        if (!mbar_wait(&bars[s], parity)) {
            failed = true;
            failed_at = it;
            break;
        }
        __syncwarp();   // zero rows written by other lanes are visible from here on
        const int r0 = j_begin + (warp + it * kWarps) * kTileRows;
        const uint32_t st = ring_u32 + s * kStageBytes;

        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4(st + k_off + kk * 32, a0, a1, a2, a3);
            mma_bf16_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
        }
        const bool v0 = (r0 + gid) < lim;
        const bool v1 = (r0 + gid + 8) < lim;
        sc[0] = v0 ? sc[0] * p.scale_log2 : -INFINITY;
        sc[1] = v0 ? sc[1] * p.scale_log2 : -INFINITY;
        sc[2] = v1 ? sc[2] * p.scale_log2 : -INFINITY;
        sc[3] = v1 ? sc[3] * p.scale_log2 : -INFINITY;

        float t0 = fmaxf(sc[0], sc[2]);
        float t1 = fmaxf(sc[1], sc[3]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, off));
            t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, off));
        }
        const float n0 = fmaxf(m0, t0);
        const float n1 = fmaxf(m1, t1);
        const float u0 = (n0 == -INFINITY) ? 0.f : n0;
        const float u1 = (n1 == -INFINITY) ? 0.f : n1;
        const float alpha0 = fast_exp2(m0 - u0);
        const float alpha1 = fast_exp2(m1 - u1);
        m0 = n0;
        m1 = n1;

        const __nv_bfloat162 p01 = __floats2bfloat162_rn(fast_exp2(sc[0] - u0), fast_exp2(sc[1] - u1));
        const __nv_bfloat162 p23 = __floats2bfloat162_rn(fast_exp2(sc[2] - u0), fast_exp2(sc[3] - u1));
        // the sums use the same bf16-rounded weights that multiply V
        l0 = l0 * alpha0 + __low2float(p01) + __low2float(p23);
        l1 = l1 * alpha1 + __high2float(p01) + __high2float(p23);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            acc[mt][0] *= alpha0;
            acc[mt][1] *= alpha1;
            acc[mt][2] *= alpha0;
            acc[mt][3] *= alpha1;
        }
        const uint32_t pb0 = movmatrix_t(*reinterpret_cast<const uint32_t*>(&p01));
        const uint32_t pb1 = movmatrix_t(*reinterpret_cast<const uint32_t*>(&p23));
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            uint32_t a0, a1, a2, a3;
            ldsm_x4_t(st + v_off + mt * 32, a0, a1, a2, a3);
            mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
        }
        __syncwarp();
        if (it + kStages < my_tiles) {
            const int rn = j_begin + (warp + (it + kStages) * kWarps) * kTileRows;
            issue_tile(ring + s * kStageBytes, &bars[s], kbase, vbase, row_stride, rn,
                       min(kTileRows, j_end - rn), lane);
        }
    }
    if (failed) {
        // Drain this warp's other copies in flight, with the same bound: tiles
        // 0 .. issued-1 were issued; wait for the last one of each stage.
        const int issued = min(my_tiles, failed_at + kStages);
        for (int s = 0; s < kStages; ++s) {
            int last = -1;
            for (int i = s; i < issued; i += kStages) last = i;
            if (last >= 0) (void)mbar_wait(&bars[s], static_cast<uint32_t>((last / kStages) & 1));
        }
        if (lane == 0) {
            s_failed = 1;
            report(p.status, ARK_DEV_TIMEOUT);
        }
    }

    // full per-head sums of this warp
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }

    __syncthreads();   // rings are free: reuse them as the merge area
    float* o_s = reinterpret_cast<float*>(smem);                       // [warp][head][dim]
    float* ml_s = o_s + kWarps * kGroup * kHeadDim;                    // [warp][head][2]
    {
        float* ow = o_s + warp * kGroup * kHeadDim;
        const int h0 = 2 * tig, h1 = 2 * tig + 1;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
            const int d = 16 * mt + gid;
            ow[h0 * kHeadDim + d] = acc[mt][0];
            ow[h1 * kHeadDim + d] = acc[mt][1];
            ow[h0 * kHeadDim + d + 8] = acc[mt][2];
            ow[h1 * kHeadDim + d + 8] = acc[mt][3];
        }
        if (gid == 0) {
            float* mw = ml_s + warp * kGroup * 2;
            mw[h0 * 2] = m0;  mw[h0 * 2 + 1] = l0;
            mw[h1 * 2] = m1;  mw[h1 * 2 + 1] = l1;
        }
    }
    __syncthreads();
    if (s_failed) return;

    {
        const int h = threadIdx.x >> 4;          // 0..7
        const int d0 = (threadIdx.x & 15) * 8;   // 8 dims per thread
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, ml_s[(w * kGroup + h) * 2]);
        float e[kWarps];
        float lsum = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = ml_s[(w * kGroup + h) * 2];
            e[w] = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
            lsum += e[w] * ml_s[(w * kGroup + h) * 2 + 1];
        }
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            if (e[w] == 0.f) continue;
            const float4* src = reinterpret_cast<const float4*>(o_s + (w * kGroup + h) * kHeadDim + d0);
            const float4 x0 = src[0], x1 = src[1];
            o[0] += e[w] * x0.x; o[1] += e[w] * x0.y; o[2] += e[w] * x0.z; o[3] += e[w] * x0.w;
            o[4] += e[w] * x1.x; o[5] += e[w] * x1.y; o[6] += e[w] * x1.z; o[7] += e[w] * x1.w;
        }
        const bool empty = (M == -INFINITY);
        const float inv = empty ? 0.f : 1.f / lsum;
        const float lse = empty ? -INFINITY : (M + __log2f(lsum)) * kLn2;
        const size_t bh = static_cast<size_t>(b) * p.Hq + head0 + h;
        if (p.nsplit == 1) {
            uint4 packed;
            packed.x = pack_bf16x2(o[0] * inv, o[1] * inv);
            packed.y = pack_bf16x2(o[2] * inv, o[3] * inv);
            packed.z = pack_bf16x2(o[4] * inv, o[5] * inv);
            packed.w = pack_bf16x2(o[6] * inv, o[7] * inv);
            *reinterpret_cast<uint4*>(L.o + bh * kHeadDim + d0) = packed;
            if ((threadIdx.x & 15) == 0) L.lse[bh] = lse;
        } else {
            if (!empty) {
                float4* dst = reinterpret_cast<float4*>(L.o_part + (bh * p.nsplit + split) * kHeadDim + d0);
                dst[0] = make_float4(o[0] * inv, o[1] * inv, o[2] * inv, o[3] * inv);
                dst[1] = make_float4(o[4] * inv, o[5] * inv, o[6] * inv, o[7] * inv);
            }
            if ((threadIdx.x & 15) == 0) L.lse_part[bh * p.nsplit + split] = lse;
        }
    }
}

// One warp per (b, h): merge nsplit normalised partials by log-sum-exp.
__global__ void __launch_bounds__(128) combine_kernel(const __grid_constant__ CombineParams p) {
    const int warp_global = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (warp_global >= p.B * p.Hq) return;
    const CombineLayer& L = p.layer[blockIdx.y];
    const size_t bh = static_cast<size_t>(warp_global);
    const float* lp = L.lse_part + bh * p.nsplit;
    float M = -INFINITY;
    for (int c = lane; c < p.nsplit; c += 32) M = fmaxf(M, lp[c]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float wsum = 0.f;
    if (M != -INFINITY) {
        for (int c = 0; c < p.nsplit; ++c) {
            const float lc = lp[c];
            if (lc == -INFINITY) continue;
            const float w = __expf(lc - M);
            wsum += w;
            const float4 x = reinterpret_cast<const float4*>(L.o_part + (bh * p.nsplit + c) * kHeadDim)[lane];
            acc.x += w * x.x; acc.y += w * x.y; acc.z += w * x.z; acc.w += w * x.w;
        }
    }
    const bool empty = (M == -INFINITY);
    const float inv = empty ? 0.f : 1.f / wsum;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(L.o + bh * kHeadDim)[lane] = packed;
    if (lane == 0) L.lse[bh] = empty ? -INFINITY : M + __logf(wsum);
}

}  // namespace ark

using namespace ark;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int decode_chunk(int T, int max_splits) {
    const int per = (T + max_splits - 1) / max_splits;
    int chunk = ((per + kTileRows - 1) / kTileRows) * kTileRows;
    if (chunk < 64) chunk = 64;
    return chunk;
}

int decode_nsplit(int T, int max_splits) {
    const int chunk = decode_chunk(T, max_splits);
    return (T + chunk - 1) / chunk;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t part_o_bytes(int B, int Hq, int D, int nsplit) {
    return align256(static_cast<size_t>(B) * Hq * nsplit * D * sizeof(float));
}

size_t part_lse_bytes(int B, int Hq, int nsplit) {
    return align256(static_cast<size_t>(B) * Hq * nsplit * sizeof(float));
}

ark_status check_decode_shape(int B, int T, int Hq, int Hkv, int D) {
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return ARK_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ARK_ERR_INVALID_ARG;
    if (T > ARK_MAX_T) return ARK_ERR_UNSUPPORTED;
    if (D != kHeadDim || Hq / Hkv != kGroup) return ARK_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * ARK_MAX_LAYERS > 2147483647LL) return ARK_ERR_UNSUPPORTED;
    return ARK_OK;
}

bool g_decode_attr_set = false;

ark_status ensure_decode_attr() {
    if (!g_decode_attr_set) {
        if (cudaFuncSetAttribute(decode_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 kDecodeSmem) != cudaSuccess)
            return ARK_ERR_CUDA;
        g_decode_attr_set = true;
    }
    return ARK_OK;
}

}  // namespace

extern "C" size_t ark_attn_decode_workspace_size(int B, int Hq, int D, int T, int max_splits) {
    if (B <= 0 || Hq <= 0 || D <= 0 || T <= 0 || max_splits <= 0) return 0;
    const int nsplit = decode_nsplit(T, max_splits);
    if (nsplit <= 1) return 0;
    return part_o_bytes(B, Hq, D, nsplit) + part_lse_bytes(B, Hq, nsplit);
}

extern "C" ark_status ark_attn_decode(const void* q, const void* cache_k, const void* cache_v,
                                      const int32_t* kv_len, int B, int T, int Hq, int Hkv, int D,
                                      float scale, ark_decode_mode mode, int max_splits,
                                      void* workspace, size_t workspace_bytes,
                                      void* o, float* lse, uint32_t* d_status, cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !kv_len || !o || !lse) return ARK_ERR_INVALID_ARG;
    ark_status st = check_decode_shape(B, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (max_splits <= 0 || !(scale > 0.f) || (mode != ARK_LENGTH_AWARE && mode != ARK_MASKED_STATIC))
        return ARK_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return ARK_ERR_INVALID_ARG;
    const int chunk = decode_chunk(T, max_splits);
    const int nsplit = (T + chunk - 1) / chunk;
    const size_t need = ark_attn_decode_workspace_size(B, Hq, D, T, max_splits);
    if (need > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace))) return ARK_ERR_WORKSPACE;
    if ((st = ensure_decode_attr()) != ARK_OK) return st;

    DecodeParams prm{};
    prm.kv_len = kv_len;
    prm.status = d_status;
    prm.B = B; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    prm.nsplit = nsplit;
    prm.chunk = chunk;
    prm.masked = (mode == ARK_MASKED_STATIC) ? 1 : 0;
    prm.scale_log2 = scale * kLog2e;
    float* o_part = nullptr;
    float* lse_part = nullptr;
    if (nsplit > 1) {
        o_part = static_cast<float*>(workspace);
        lse_part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + part_o_bytes(B, Hq, D, nsplit));
    }
    prm.layer[0] = DecodeLayer{static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(cache_k),
                               static_cast<const uint16_t*>(cache_v), static_cast<uint16_t*>(o), lse,
                               o_part, lse_part};
    dim3 grid(nsplit, Hkv, B);
    decode_split_kernel<<<grid, kWarps * 32, kDecodeSmem, stream>>>(prm);
    if (cudaGetLastError() != cudaSuccess) return ARK_ERR_CUDA;
    if (nsplit > 1) {
        CombineParams cp{};
        cp.B = B; cp.Hq = Hq; cp.nsplit = nsplit;
        cp.layer[0] = CombineLayer{o_part, lse_part, static_cast<uint16_t*>(o), lse};
        dim3 cgrid((B * Hq + 3) / 4, 1);
        combine_kernel<<<cgrid, 128, 0, stream>>>(cp);
        if (cudaGetLastError() != cudaSuccess) return ARK_ERR_CUDA;
    }
    return ARK_OK;
}

extern "C" ark_status ark_attn_combine(const float* o_part, const float* lse_part, int B, int Hq,
                                       int nsplit, int D, void* o, float* lse, cudaStream_t stream) {
    if (!o_part || !lse_part || !o || !lse) return ARK_ERR_INVALID_ARG;
    if (B <= 0 || Hq <= 0 || nsplit <= 0 || D <= 0) return ARK_ERR_INVALID_ARG;
    if (D != kHeadDim) return ARK_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * Hq > 2147483647LL / 4) return ARK_ERR_UNSUPPORTED;
    if (!aligned16(o_part) || !aligned16(o) || (reinterpret_cast<uintptr_t>(lse_part) & 3u) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return ARK_ERR_INVALID_ARG;
    CombineParams cp{};
    cp.B = B; cp.Hq = Hq; cp.nsplit = nsplit;
    cp.layer[0] = CombineLayer{o_part, lse_part, static_cast<uint16_t*>(o), lse};
    dim3 cgrid((B * Hq + 3) / 4, 1);
    combine_kernel<<<cgrid, 128, 0, stream>>>(cp);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}
