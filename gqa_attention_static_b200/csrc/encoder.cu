// encoder.cu -- bidirectional (non-causal) multi-head attention of the audio
// encoder, on the 5th-generation tensor cores.
//
// ARK-ASR-3B's audio tower is a Whisper-style encoder with rotary self-
// attention ("Inside ARK-ASR-3B's Whisper and Qwen architecture", components
// list; "ARK-ASR-3B -- INT8 ONNX", Inference step 1: the encoder maps the mel
// frames of one clip to [seq, 1280]).  The pages give neither the head count
// nor the rotary parameters of that encoder; reading taken: the Whisper-large
// geometry that a 1280-wide model has (20 heads of 64 dims), plain multi-head
// attention in which every frame of a clip attends to every frame of the same
// clip, q and k already rotated by the caller.  Clips are up to 30 s
// (1500 frames after the stride-2 convolution; the 30-second Whisper boundary
// of the SGLang-Omni cookbook's audio handling) and are encoded in batches of
// up to 8 (its encoder_max_batch_size).
//
// Per (clip b, head h, row i < len[b]):
//   o[b,i,h,:] = sum_{j < len[b]} softmax_j(scale <q[b,i,h,:], k[b,j,h,:]>) v[b,j,h,:]
//   lse[b,h,i] = ln sum_{j < len[b]} exp(scale <q[b,i,h,:], k[b,j,h,:]>)
//
// Tiling: one CTA per 128 consecutive frames of one (clip, head); Q tile
// 128 x 64 (16 KB, one TMA box, 128-byte swizzle), K and V blocks of 64 frames
// (8 KB each) through 4-stage rings.  S = Q K^T is 4 MMAs of 128x64x16 into a
// double-buffered TMEM S; P (bf16) is stored back over S and O += P V is 4 MMAs
// of 128x64x16 with P read from TMEM and V an MN-major operand.  Warp roles as
// in the prefill kernel: warp 0 TMA, warp 1 MMA (one thread), warps 2..9
// softmax, two threads per row (32 keys of a block each), row maxima traded
// through shared memory behind an AND-reducing named barrier; lazily rescaled
// O; keys past len[b] are masked (and their V rows zeroed) in the last block
// only.  Rows past len[b] are computed on whatever q holds and not written.
#include "common.cuh"
#include "tma_host.h"

namespace ark {
namespace enc {

constexpr int kRows = 128;               // frames per tile (MMA M)
constexpr int kD = 64;                   // head dim
constexpr int kBN = 64;                  // keys per block
constexpr int kQBytes = kRows * 128;     // 128 rows x 64 dims bf16
constexpr int kKV = kBN * 128;           // a K or V block (8 KB)
constexpr int kThreads = 320;
constexpr int kSoftmaxThreads = 256;
constexpr int kKStages = 4;
constexpr int kVStages = 4;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kKStages * kKV;
constexpr int kOffBar = kOffV + kVStages * kKV;
constexpr int kBarQ = 0;
constexpr int kBarKFull = 1;
constexpr int kBarKEmpty = kBarKFull + kKStages;
constexpr int kBarVFull = kBarKEmpty + kKStages;
constexpr int kBarVEmpty = kBarVFull + kVStages;
constexpr int kBarSFull = kBarVEmpty + kVStages;   // 2
constexpr int kBarPFull = kBarSFull + 2;           // 2
constexpr int kBarPvDone = kBarPFull + 2;
constexpr int kNumBars = kBarPvDone + 1;
constexpr int kOffXchg = kOffBar + kNumBars * 8;   // [3][2][128] fp32
constexpr int kOffTmemPtr = kOffXchg + 3 * 2 * kRows * 4;
constexpr int kOffFlag = kOffTmemPtr + 8;
constexpr int kSmemBytes = kOffFlag + 16;

constexpr uint32_t kColS = 0;            // S buffers: 0..63, 64..127
constexpr uint32_t kColO = 128;          // O: 128..191
constexpr uint32_t kTmemCols = 256;

constexpr uint32_t kIdescF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescF16 | ((64u >> 3) << 17);                // N = 64 keys, K-major B
constexpr uint32_t kIdescPV = kIdescF16 | ((64u >> 3) << 17) | (1u << 16);   // N = 64 dims, MN-major B

constexpr float kLazyRescale = 8.0f;

struct Params {
    CUtensorMap qmap;    // q as (64, H, B*S), box (64, 1, 128)
    CUtensorMap kmap;    // k as (64, H, B*S), box (64, 1, 64)
    CUtensorMap vmap;
    uint16_t* o;         // [B, S, H, 64]
    float* lse;          // [B, H, S]
    const int32_t* len;
    uint32_t* status;
    int B, S, H, QT;
    float scale_log2;
};

}  // namespace enc

__device__ __forceinline__ bool enc_bar_and_all(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, %2, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(out) : "r"(static_cast<uint32_t>(pred)), "n"(enc::kSoftmaxThreads) : "memory");
    return out != 0;
}

__global__ void __launch_bounds__(enc::kThreads, 2) encoder_attn_kernel(const __grid_constant__ enc::Params p) {
    using namespace enc;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int qt = blockIdx.x % p.QT;
    const int h = (blockIdx.x / p.QT) % p.H;
    const int b = blockIdx.x / (p.QT * p.H);
    int len = __ldg(p.len + b);
    if (len < 0 || len > p.S) {
        if (threadIdx.x == 0 && qt == 0 && h == 0) report(p.status, ARK_DEV_BAD_KVLEN);
        len = len < 0 ? 0 : p.S;
    }
    const int t0 = qt * kRows;
    if (t0 >= len) return;                                   // whole CTA: no live row
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) report(p.status, ARK_DEV_TIMEOUT);
        return;
    }
    const int nblk = (len + kBN - 1) / kBN;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + kOffFlag);
    const int row0 = b * p.S;                                // first row of the clip

    auto load_k = [&](int j) {
        const int ks = j % kKStages;
        mbar_arrive_expect_tx(&bars[kBarKFull + ks], kKV);
        tma_load_3d(smem + kOffK + ks * kKV, &p.kmap, 0, h, row0 + j * kBN, &bars[kBarKFull + ks]);
    };
    auto load_v = [&](int j) {
        const int vs = j % kVStages;
        mbar_arrive_expect_tx(&bars[kBarVFull + vs], kKV);
        tma_load_3d(smem + kOffV + vs * kKV, &p.vmap, 0, h, row0 + j * kBN, &bars[kBarVFull + vs]);
    };
    constexpr int kPre = 4;
    static_assert(kKStages >= kPre && kVStages >= kPre, "preloaded blocks need their own stages");
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(&bars[i], (i == kBarPFull || i == kBarPFull + 1) ? kSoftmaxThreads : 1);
        *failed_flag = 0;
        fence_mbar_init();
        mbar_arrive_expect_tx(&bars[kBarQ], kQBytes);
        tma_load_3d(smem + kOffQ, &p.qmap, 0, h, row0 + t0, &bars[kBarQ]);
        for (int j = 0; j < min(nblk, kPre); ++j) {
            load_k(j);
            load_v(j);
        }
    }
    if (warp == 0) tmem_alloc(tmem_ptr, kTmemCols);
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            bool ok = true;
            for (int j = kPre; j < nblk; ++j) {
                if (!mbar_wait(&bars[kBarKEmpty + j % kKStages], ((j / kKStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                load_k(j);
                if (!mbar_wait(&bars[kBarVEmpty + j % kVStages], ((j / kVStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                load_v(j);
            }
            if (!ok) {
                atomicExch(failed_flag, 1);
                report(p.status, ARK_DEV_TIMEOUT);
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQ], 0));
        auto wait_k = [&](int j) {
            return __all_sync(0xffffffffu, mbar_wait(&bars[kBarKFull + j % kKStages], (j / kKStages) & 1));
        };
        auto wait_v = [&](int j) {
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarVFull + j % kVStages], (j / kVStages) & 1)))
                return false;
            const int live = len - j * kBN;                  // frames of the clip in this block
            if (live < kBN) {
                uint8_t* vt = smem + kOffV + (j % kVStages) * kKV;
                for (int i = lane; i < (kBN - live) * 8; i += 32)
                    *reinterpret_cast<uint4*>(vt + (live + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            __syncwarp();
            return true;
        };
        auto issue_qk = [&](int j) {
            if (lane == 0) {
                tc_fence_after();
                const uint32_t d = tmem + kColS + (j & 1) * kBN;
                const uint32_t kb = sbase + kOffK + (j % kKStages) * kKV;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(d, umma_desc_sw128(sbase + kOffQ + kk * 32, 16, 1024), umma_desc_sw128(kb + kk * 32, 16, 1024),
                             kIdescQK, kk > 0 ? 1u : 0u);
                umma_commit(&bars[kBarSFull + (j & 1)]);
                umma_commit(&bars[kBarKEmpty + j % kKStages]);
            }
            __syncwarp();
        };
        auto issue_pv = [&](int j) {
            if (lane == 0) {
                tc_fence_after();
                const uint32_t pa = tmem + kColS + (j & 1) * kBN;
                const uint32_t vb = sbase + kOffV + (j % kVStages) * kKV;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16_ts(tmem + kColO, pa + kk * 8, umma_desc_sw128(vb + kk * 16 * 128, kKV, 1024), kIdescPV,
                                (j > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&bars[kBarVEmpty + j % kVStages]);
                umma_commit(&bars[kBarPvDone]);
            }
            __syncwarp();
        };
        if (ok) ok = wait_k(0);
        if (ok) issue_qk(0);
        for (int j = 0; j < nblk && ok; ++j) {
            if (j + 1 < nblk) {
                if (!(ok = wait_k(j + 1))) break;
                issue_qk(j + 1);
            }
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPFull + (j & 1)], (j >> 1) & 1)))) break;
            if (!(ok = wait_v(j))) break;
            issue_pv(j);
        }
        if (!ok && lane == 0) {
            atomicExch(failed_flag, 1);
            report(p.status, ARK_DEV_TIMEOUT);
        }
    } else {
        // ================================================= softmax + epilogue
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;               // keys 32*half .. +31 of a block; dims 32*half .. +31 of o
        const int r = quad * 32 + lane;                 // this thread's row (frame t0 + r)
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        float* xchg = reinterpret_cast<float*>(smem + kOffXchg);
        float m_ref = -INFINITY, e_sum = 0.f, r_sum = 0.f;
        bool ok = true;
        // every tcgen05.ld/st is .sync.aligned and sits on warp-uniform control flow;
        // the loop is left by all 256 softmax threads together (AND-reduced exit test)
        for (int j = 0; j < nblk; ++j) {
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars[kBarSFull + (j & 1)], (j >> 1) & 1));
            tc_fence_after();
            const int nvalid = min(32, len - j * kBN - half * 32);   // keys of this half inside the clip
            uint32_t v[32];
            tmem_ld32(lane_base + kColS + (j & 1) * kBN + half * 32, v);
            tmem_wait_ld();
            float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            if (nvalid >= 32) {
#pragma unroll
                for (int i = 0; i < 32; ++i) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(v[i]));
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nvalid) m4[i & 3] = fmaxf(m4[i & 3], __uint_as_float(v[i]));
            }
            const float my_max = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
            float* xm = xchg + (j & 1) * 2 * kRows;
            xm[half * kRows + r] = my_max;
            if (!enc_bar_and_all(ok)) {
                ok = false;
                break;
            }
            const float bm = fmaxf(my_max, xm[(half ^ 1) * kRows + r]) * p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (m_ref == -INFINITY) {
                m_ref = bm;
            } else if (bm > m_ref + kLazyRescale) {
                alpha = fast_exp2(m_ref - bm);
                m_ref = bm;
                rescale = true;
            }
            const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
            if (__any_sync(0xffffffffu, rescale)) {
                if (j >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone], (j - 1) & 1));
                tc_fence_after();
                e_sum *= alpha;
                r_sum *= alpha;
#pragma unroll
                for (int c = 0; c < 2; ++c) {         // this half rescales O columns 32*half .. +31
                    uint32_t o[16];
                    tmem_ld16(lane_base + kColO + half * 32 + c * 16, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st16(lane_base + kColO + half * 32 + c * 16, o);
                }
                tmem_wait_st();
            }
            const bool full = nvalid >= 32;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
                const float x0 = __uint_as_float(v[i]) * p.scale_log2 - mu;
                const float x1 = __uint_as_float(v[i + 1]) * p.scale_log2 - mu;
                const float s0 = (full || i < nvalid) ? fast_exp2(x0) : 0.f;
                const float s1 = (full || i + 1 < nvalid) ? fast_exp2(x1) : 0.f;
                const __nv_bfloat162 pb = __floats2bfloat162_rn(s0, s1);
                e_sum += s0 + s1;
                const float2 pf2 = __bfloat1622float2(pb);
                r_sum += pf2.x + pf2.y;
                pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&pb);
            }
            tmem_st16(lane_base + kColS + (j & 1) * kBN + half * 16, pk);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bars[kBarPFull + (j & 1)]);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone], (nblk - 1) & 1));
        tc_fence_after();
        float* xs = xchg + 2 * 2 * kRows;
        xs[half * kRows + r] = e_sum;
        ok = enc_bar_and_all(ok);
        const float e_tot = e_sum + xs[(half ^ 1) * kRows + r];
        ok = enc_bar_and_all(ok);
        xs[half * kRows + r] = r_sum;
        ok = enc_bar_and_all(ok);
        const float r_tot = r_sum + xs[(half ^ 1) * kRows + r];
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        } else {
            const int t = t0 + r;
            const bool live = t < len;
            const float inv = 1.f / r_tot;
            uint4* orow = reinterpret_cast<uint4*>(
                p.o + ((static_cast<size_t>(row0) + t) * p.H + h) * kD + half * 32);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t o[16];
                tmem_ld16(lane_base + kColO + half * 32 + c * 16, o);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
                        orow[2 * c + q] = w;
                    }
                }
            }
            if (live && half == 0)
                p.lse[(static_cast<size_t>(b) * p.H + h) * p.S + t] = (m_ref + __log2f(e_tot)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        if (*failed_flag) {
            for (int s = 0; s < kKStages; ++s) (void)mbar_wait(&bars[kBarKFull + s], 0);
            for (int s = 0; s < kVStages; ++s) (void)mbar_wait(&bars[kBarVFull + s], 0);
            (void)mbar_wait(&bars[kBarPvDone], (nblk - 1) & 1);
        }
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace ark

using namespace ark;

namespace {

bool enc_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool g_encoder_attr[64];

}  // namespace

extern "C" ark_status ark_attn_encoder(const void* q, const void* k, const void* v, const int32_t* len, int B, int S,
                                       int H, int D, float scale, void* o, float* lse, uint32_t* d_status,
                                       cudaStream_t stream) {
    if (!q || !k || !v || !len || !o || !lse) return ARK_ERR_INVALID_ARG;
    if (B <= 0 || S <= 0 || H <= 0 || D <= 0 || !(scale > 0.f)) return ARK_ERR_INVALID_ARG;
    if (D != enc::kD) return ARK_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * S >= (1LL << 31) || H > 65535) return ARK_ERR_UNSUPPORTED;
    if (!enc_aligned16(q) || !enc_aligned16(k) || !enc_aligned16(v) || !enc_aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return ARK_ERR_INVALID_ARG;
    enc::Params prm{};
    const long long rows = static_cast<long long>(B) * S;
    if (!hd64_tensor_map(&prm.qmap, q, rows, H, enc::kRows) || !hd64_tensor_map(&prm.kmap, k, rows, H, enc::kBN) ||
        !hd64_tensor_map(&prm.vmap, v, rows, H, enc::kBN))
        return ARK_ERR_CUDA;
    prm.o = static_cast<uint16_t*>(o);
    prm.lse = lse;
    prm.len = len;
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.H = H;
    prm.QT = (S + enc::kRows - 1) / enc::kRows;
    prm.scale_log2 = scale * kLog2e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    if (!g_encoder_attr[dev]) {
        if (cudaFuncSetAttribute(encoder_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, enc::kSmemBytes) !=
            cudaSuccess)
            return ARK_ERR_CUDA;
        g_encoder_attr[dev] = true;
    }
    const long long ctas = static_cast<long long>(B) * H * prm.QT;
    if (ctas >= (1LL << 31)) return ARK_ERR_UNSUPPORTED;
    encoder_attn_kernel<<<static_cast<unsigned>(ctas), enc::kThreads, enc::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}
