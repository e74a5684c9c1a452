// qkv_proj.cu -- the Q/K/V projections of a decoder layer on the tcgen05
// tensor cores, with RoPE and the delta write into the static cache fused
// into the epilogue.
//
// "ARK-ASR-3B -- INT8 ONNX" model card: a Qwen2 decoder with hidden 2048, 16
// query heads and 2 KV heads of 128 dims; each call's new key/value rows go
// into cache_{key,value}_i at cache_position (section Shapes).  The three
// projections are one Linear over the concatenated weight W = [Wq; Wk; Wv]
// ([N, K], N = (Hq + 2 Hkv) * 128, K = hidden) with an optional bias:
//   p[m, n] = bf16( sum_k x[m, k] W[n, k] + bias[n] )
// and the fused form goes on, per token row m = (request b, row t < n_new[b])
// at position pos = pos0[b] + t, to rotate the q and k heads (Qwen2
// rotate-half RoPE, the same table and the same double-precision formula as
// ark_attn_append_rope) and to store q, and k and v into the caches at pos.
//
// Tiling: one CTA per (128 token rows, one head = 128 output features).  The
// K dimension streams through a 4-stage ring of 64-wide chunks (x tile 16 KB,
// W tile 16 KB, 128-byte swizzle) loaded by TMA; one thread issues 4 MMAs of
// 128x128x16 per chunk into a 128-column TMEM accumulator.  Epilogue: 4 warps,
// one token row per thread, so the rotary partners i and i + 64 of a head are
// in the same thread.  The projection value is the fp32 accumulator plus the
// bias, added in double and rounded once to bf16; the rotation then works on
// that bf16 value exactly as the append kernel does, so the fused result is
// bit-identical to ark_attn_qkv_proj followed by ark_attn_append_rope.
#include "common.cuh"
#include "tma_host.h"

namespace ark {
namespace qp {

constexpr int kBM = 128;                 // token rows per tile (MMA M)
constexpr int kBN = 128;                 // output features per tile: one head (MMA N)
constexpr int kBK = 64;                  // K chunk: 64 bf16 = one 128-byte swizzle row
constexpr int kStages = 4;
constexpr int kTileA = kBM * 128;        // 16 KB
constexpr int kTileB = kBN * 128;        // 16 KB
constexpr int kStageBytes = kTileA + kTileB;
constexpr int kThreads = 192;            // warp 0: TMA, warp 1: MMA, warps 2..5: epilogue

constexpr int kOffBar = kStages * kStageBytes;
constexpr int kBarFull = 0;              // [kStages]
constexpr int kBarEmpty = kBarFull + kStages;
constexpr int kBarDone = kBarEmpty + kStages;
constexpr int kNumBars = kBarDone + 1;
constexpr int kOffTmemPtr = kOffBar + kNumBars * 8;
constexpr int kOffFlag = kOffTmemPtr + 8;
constexpr int kSmemBytes = kOffFlag + 8;
constexpr uint32_t kTmemCols = 128;

// kind::f16, bf16 x bf16 -> fp32, M = 128, N = 128, A and B K-major
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct Params {
    CUtensorMap xmap;          // x [M][K] as (K, M), box (64, 128)
    CUtensorMap wmap;          // W [N][K] as (K, N), box (64, 128)
    const uint16_t* bias;      // [N] or null
    int M, K, N;
    int fused;                 // 0: p -> out [M][N]; 1: RoPE + delta write
    uint16_t* out;
    uint16_t* q;               // [B, S, Hq, 128]
    uint16_t* cache_k;         // [B, T, Hkv, 128]
    uint16_t* cache_v;
    const int32_t* pos0;
    const int32_t* n_new;
    const float2* table;       // [T][64] {cos, sin}
    uint32_t* status;
    int B, S, T, Hq, Hkv;
};

}  // namespace qp

__global__ void __launch_bounds__(qp::kThreads, 1) qkv_proj_kernel(const __grid_constant__ qp::Params p) {
    using namespace qp;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int head = blockIdx.x;                 // output features 128*head .. +127
    const int m0 = blockIdx.y * kBM;
    const int nk = p.K / kBK;
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) report(p.status, ARK_DEV_TIMEOUT);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + kOffFlag);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], 1);
        *failed_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_ptr, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            int last = -1;
            bool ok = true;
            for (int c = 0; c < nk; ++c) {
                const int st = c % kStages;
                if (c >= kStages && !(ok = mbar_wait(&bars[kBarEmpty + st], ((c / kStages) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[kBarFull + st], kStageBytes);
                tma_load_2d(smem + st * kStageBytes, &p.xmap, c * kBK, m0, &bars[kBarFull + st]);
                tma_load_2d(smem + st * kStageBytes + kTileA, &p.wmap, c * kBK, head * kBN, &bars[kBarFull + st]);
                last = c;
            }
            if (!ok) {
                atomicExch(failed_flag, 1);
                report(p.status, ARK_DEV_TIMEOUT);
            }
            // the copies of the last kStages chunks have landed before the shared memory can go away
            for (int c = last - kStages + 1; c <= last; ++c)
                if (c >= 0) (void)mbar_wait(&bars[kBarFull + c % kStages], (c / kStages) & 1);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        bool ok = true;
        for (int c = 0; c < nk; ++c) {
            const int st = c % kStages;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarFull + st], (c / kStages) & 1)))) break;
            if (lane == 0) {
                tc_fence_after();
                const uint32_t a = sbase + st * kStageBytes;
                const uint32_t b = a + kTileA;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(tmem, umma_desc_sw128(a + kk * 32, 16, 1024), umma_desc_sw128(b + kk * 32, 16, 1024),
                             kIdesc, (c > 0 || kk > 0) ? 1u : 0u);
                umma_commit(&bars[kBarEmpty + st]);
            }
            __syncwarp();
        }
        if (!ok) {
            atomicExch(failed_flag, 1);                  // before the commit the epilogue waits on
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        }
        __syncwarp();
        if (lane == 0) umma_commit(&bars[kBarDone]);     // also when the loop gave up: MMAs issued so far
        __syncwarp();
    } else {
        // ================================================= epilogue: one token row per thread
        const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
        const int r = quad * 32 + lane;
        const int m = m0 + r;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarDone], 0)) &&
                        !*reinterpret_cast<volatile int*>(failed_flag);
        tc_fence_after();
        if (!ok) {
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        } else if (!p.fused) {
            // p = bf16(acc + bias) -> out[m][128*head ..]
            uint16_t* dst = p.out + static_cast<size_t>(m) * p.N + head * kBN;
            for (int c16 = 0; c16 < kBN / 16; ++c16) {
                uint32_t a[16];
                tmem_ld16(lane_base + c16 * 16, a);
                tmem_wait_ld();
                if (m < p.M) {
                    uint32_t w[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int n = head * kBN + c16 * 16 + 2 * i;
                        const double b0 = p.bias ? bf16_bits_to_f64(p.bias[n]) : 0.0;
                        const double b1 = p.bias ? bf16_bits_to_f64(p.bias[n + 1]) : 0.0;
                        w[i] = static_cast<uint32_t>(f64_to_bf16_rn(static_cast<double>(__uint_as_float(a[2 * i])) + b0)) |
                               (static_cast<uint32_t>(f64_to_bf16_rn(static_cast<double>(__uint_as_float(a[2 * i + 1])) + b1)) << 16);
                    }
                    uint4* d4 = reinterpret_cast<uint4*>(dst + c16 * 16);
                    d4[0] = make_uint4(w[0], w[1], w[2], w[3]);
                    d4[1] = make_uint4(w[4], w[5], w[6], w[7]);
                }
            }
        } else {
            // which row of which request, and where it goes
            uint16_t* dst = nullptr;
            bool rotate = false;
            int pos = 0;
            if (m < p.M) {
                const int b = m / p.S, t = m - b * p.S;
                int nn = __ldg(p.n_new + b);
                if (nn < 0 || nn > p.S) {
                    if (t == 0 && head == 0) report(p.status, ARK_DEV_BAD_KVLEN);
                    nn = nn < 0 ? 0 : p.S;
                }
                pos = __ldg(p.pos0 + b) + t;
                if (t < nn) {
                    if (pos < 0 || pos >= p.T) {
                        if (head == 0) report(p.status, ARK_DEV_BAD_POS);
                    } else if (head < p.Hq) {
                        dst = p.q + (static_cast<size_t>(m) * p.Hq + head) * kHeadDim;
                        rotate = true;
                    } else if (head < p.Hq + p.Hkv) {
                        dst = p.cache_k + ((static_cast<size_t>(b) * p.T + pos) * p.Hkv + (head - p.Hq)) * kHeadDim;
                        rotate = true;
                    } else {
                        dst = p.cache_v +
                              ((static_cast<size_t>(b) * p.T + pos) * p.Hkv + (head - p.Hq - p.Hkv)) * kHeadDim;
                    }
                }
            }
            const float4* trow = reinterpret_cast<const float4*>(p.table + static_cast<size_t>(rotate ? pos : 0) * 64);
            // rotary pairs (i, i + 64) for i in 16-wide groups; every warp runs every tcgen05.ld
            for (int g16 = 0; g16 < 4; ++g16) {
                uint32_t lo[16], hi[16];
                tmem_ld16(lane_base + g16 * 16, lo);
                tmem_ld16(lane_base + 64 + g16 * 16, hi);
                tmem_wait_ld();
                if (!dst) continue;
                uint16_t yl[16], yh[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int d = g16 * 16 + i;
                    const int n = head * kBN + d;
                    const double bl = p.bias ? bf16_bits_to_f64(p.bias[n]) : 0.0;
                    const double bh = p.bias ? bf16_bits_to_f64(p.bias[n + 64]) : 0.0;
                    // the projection output (the Linear's bf16 value)
                    const uint16_t xl = f64_to_bf16_rn(static_cast<double>(__uint_as_float(lo[i])) + bl);
                    const uint16_t xh = f64_to_bf16_rn(static_cast<double>(__uint_as_float(hi[i])) + bh);
                    if (rotate) {
                        const float4 cs = __ldg(trow + (d >> 1));        // {c, s} of pairs d & ~1 and d | 1
                        const double c = static_cast<double>((d & 1) ? cs.z : cs.x);
                        const double s = static_cast<double>((d & 1) ? cs.w : cs.y);
                        const double a = bf16_bits_to_f64(xl);
                        const double h = bf16_bits_to_f64(xh);
                        // both products are exact in double, so contraction cannot change the result
                        yl[i] = f64_to_bf16_rn(a * c - h * s);
                        yh[i] = f64_to_bf16_rn(h * c + a * s);
                    } else {
                        yl[i] = xl;
                        yh[i] = xh;
                    }
                }
                uint32_t wl[8], wh[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    wl[i] = static_cast<uint32_t>(yl[2 * i]) | (static_cast<uint32_t>(yl[2 * i + 1]) << 16);
                    wh[i] = static_cast<uint32_t>(yh[2 * i]) | (static_cast<uint32_t>(yh[2 * i + 1]) << 16);
                }
                uint4* dl = reinterpret_cast<uint4*>(dst + g16 * 16);
                uint4* dh = reinterpret_cast<uint4*>(dst + 64 + g16 * 16);
                dl[0] = make_uint4(wl[0], wl[1], wl[2], wl[3]);
                dl[1] = make_uint4(wl[4], wl[5], wl[6], wl[7]);
                dh[0] = make_uint4(wh[0], wh[1], wh[2], wh[3]);
                dh[1] = make_uint4(wh[4], wh[5], wh[6], wh[7]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace ark

using namespace ark;

namespace {

bool qp_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool g_qp_attr[64];

ark_status launch_qkv(qp::Params& prm, const void* x, const void* w, int M, int K, int N, cudaStream_t stream) {
    if (!kmajor_tensor_map(&prm.xmap, x, M, K, qp::kBM) || !kmajor_tensor_map(&prm.wmap, w, N, K, qp::kBN))
        return ARK_ERR_CUDA;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    if (!g_qp_attr[dev]) {
        if (cudaFuncSetAttribute(qkv_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, qp::kSmemBytes) !=
            cudaSuccess)
            return ARK_ERR_CUDA;
        g_qp_attr[dev] = true;
    }
    const dim3 grid(N / qp::kBN, (M + qp::kBM - 1) / qp::kBM);
    qkv_proj_kernel<<<grid, qp::kThreads, qp::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

}  // namespace

extern "C" ark_status ark_attn_qkv_proj(const void* x, const void* w, const void* bias, int M, int K, int N,
                                        void* out, uint32_t* d_status, cudaStream_t stream) {
    if (!x || !w || !out) return ARK_ERR_INVALID_ARG;
    if (M <= 0 || K <= 0 || N <= 0 || K % qp::kBK != 0 || N % qp::kBN != 0) return ARK_ERR_INVALID_ARG;
    if (N / qp::kBN > 65535 || (M + qp::kBM - 1) / qp::kBM > 65535) return ARK_ERR_UNSUPPORTED;
    if (!qp_aligned16(x) || !qp_aligned16(w) || !qp_aligned16(out) || (reinterpret_cast<uintptr_t>(bias) & 1u))
        return ARK_ERR_INVALID_ARG;
    qp::Params prm{};
    prm.bias = static_cast<const uint16_t*>(bias);
    prm.fused = 0;
    prm.out = static_cast<uint16_t*>(out);
    prm.status = d_status;
    return launch_qkv(prm, x, w, M, K, N, stream);
}

extern "C" ark_status ark_attn_qkv_rope_append(const void* x, const void* w, const void* bias, const int32_t* pos0,
                                               const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, int D,
                                               int K, const float* d_table, void* q, void* cache_k, void* cache_v,
                                               uint32_t* d_status, cudaStream_t stream) {
    if (!x || !w || !pos0 || !n_new || !d_table || !q || !cache_k || !cache_v) return ARK_ERR_INVALID_ARG;
    if (B <= 0 || S <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || K <= 0 || K % qp::kBK != 0) return ARK_ERR_INVALID_ARG;
    if (D != kHeadDim) return ARK_ERR_UNSUPPORTED;
    const long long M = static_cast<long long>(B) * S;
    if (M >= (1LL << 31) || static_cast<long long>(B) * T >= (1LL << 31) || Hq + 2 * Hkv > 65535 ||
        (M + qp::kBM - 1) / qp::kBM > 65535)
        return ARK_ERR_UNSUPPORTED;
    if (!qp_aligned16(x) || !qp_aligned16(w) || !qp_aligned16(q) || !qp_aligned16(cache_k) ||
        !qp_aligned16(cache_v) || !qp_aligned16(d_table) || (reinterpret_cast<uintptr_t>(bias) & 1u))
        return ARK_ERR_INVALID_ARG;
    qp::Params prm{};
    prm.bias = static_cast<const uint16_t*>(bias);
    prm.fused = 1;
    prm.q = static_cast<uint16_t*>(q);
    prm.cache_k = static_cast<uint16_t*>(cache_k);
    prm.cache_v = static_cast<uint16_t*>(cache_v);
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.table = reinterpret_cast<const float2*>(d_table);
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv;
    return launch_qkv(prm, x, w, static_cast<int>(M), K, (Hq + 2 * Hkv) * kHeadDim, stream);
}
