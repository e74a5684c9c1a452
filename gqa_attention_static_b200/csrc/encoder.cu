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
// Work: a unit is 256 consecutive frames of one (clip, head), two Q tiles A
// and B of 128 rows (MMA M = 128) that share every K/V block; only units with
// a frame inside their clip exist, and tile B is skipped when it has none.
// The kernel is persistent, one CTA per SM walking the unit list (clips with
// more key blocks first) in snake order.  K and V blocks of 128 frames (16 KB
// each) stream through 3-stage TMA rings, Q through 2 buffers.
//
// Per block and tile X: S_X = Q_X K^T is 4 MMAs of 128x128x16 into 128 TMEM
// columns; the tile's softmax warpgroup (one thread per row, all 128 keys of
// the block, read in two passes of 32 keys: the row max, then the
// exponentials) stores P (bf16) in 64 TMEM columns of its own, and O_X += P_X
// V is 8 MMAs of 128x64x16 with P read from TMEM and V an MN-major operand.
// Two warps issue the MMAs, each from one thread: warp 1 the scores, warp 10
// the products.  S_X of the next block is computed as soon as the softmax has
// read the current scores out of tensor memory; before it overwrites P_X (and
// before a lazy rescale of O_X) the softmax waits for the tile's previous
// product.  Keys past len[b] get score -inf (and their V rows are zeroed) in
// the last block only.  Rows past len[b] are computed on whatever q holds and
// are not written.  Warps: 0 TMA, 1 score MMAs, 2..5 softmax of tile A, 6..9
// softmax of tile B, 10 P V MMAs.
#include "common.cuh"
#include "tma_host.h"

#include <mutex>

namespace ark {
namespace enc {

constexpr int kRows = 128;               // frames per Q tile (MMA M)
constexpr int kUnitRows = 2 * kRows;     // frames per unit (tiles A and B)
constexpr int kD = 64;                   // head dim
constexpr int kBN = 128;                 // keys per block
constexpr int kQBytes = kRows * 128;     // one Q tile: 128 rows x 64 dims bf16 (16 KB)
constexpr int kKV = kBN * 128;           // a K or V block (16 KB)
constexpr int kThreads = 352;            // warp 0 TMA, 1 score MMAs, 2..9 softmax, 10 P V MMAs
constexpr int kWgThreads = 128;          // softmax threads of one tile (one per row)
constexpr int kQStages = 2;              // units in flight (each 2 tiles)
constexpr int kStages = 3;               // K and V ring depth
constexpr int kMaxClips = 256;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQStages * 2 * kQBytes;
constexpr int kOffV = kOffK + kStages * kKV;
constexpr int kOffBar = kOffV + kStages * kKV;
constexpr int kBarQFull = 0;                       // [kQStages]
constexpr int kBarQEmpty = kBarQFull + kQStages;   // [kQStages]: every QK of the unit done
constexpr int kBarKFull = kBarQEmpty + kQStages;   // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages;    // [tile]: S_X of the next block (one phase per block)
constexpr int kBarSRead = kBarSFull + 2;           // [tile]: S_X read out by the softmax (count 128, per block)
constexpr int kBarPFull = kBarSRead + 2;           // [tile]: P_X in TMEM (count 128, one phase per block)
constexpr int kBarPvDone = kBarPFull + 2;          // [tile]: PV_X of a block done (one phase per block)
constexpr int kBarODone = kBarPvDone + 2;          // [tile]: every MMA of the unit done (one phase per unit)
constexpr int kBarOEmpty = kBarODone + 2;          // [tile]: O_X read out (count 128, one phase per unit)
constexpr int kBarDrain = kBarOEmpty + 2;          // [issuing warp]: MMAs in flight when it gives up
constexpr int kNumBars = kBarDrain + 2;
constexpr int kOffClips = kOffBar + kNumBars * 8;
//   int len[kMaxClips] (clamped), order[kMaxClips] (clips, most key blocks first), cum[kMaxClips + 1]
constexpr int kOffTmemPtr = kOffClips + (3 * kMaxClips + 1) * 4 + 12;
constexpr int kOffFlag = kOffTmemPtr + 8;
constexpr int kSmemBytes = kOffFlag + 16;
static_assert(kOffBar % 8 == 0 && kOffTmemPtr % 8 == 0, "alignment");

// TMEM columns: S_A 0..127, S_B 128..255 (fp32 scores), O_A 256..319, O_B
// 320..383, P_A 384..447, P_B 448..511 (bf16 pairs: keys 2c, 2c+1 in column c).
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;
constexpr uint32_t kColP = 384;
constexpr uint32_t kTmemCols = 512;

constexpr uint32_t kIdescF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescF16 | ((128u >> 3) << 17);               // N = 128 keys, K-major B
constexpr uint32_t kIdescPV = kIdescF16 | ((64u >> 3) << 17) | (1u << 16);   // N = 64 dims, MN-major B

constexpr float kLazyRescale = 8.0f;

struct Params {
    CUtensorMap qmap;    // q as (64, H, B*S), box (64, 1, 128)
    CUtensorMap kmap;    // k as (64, H, B*S), box (64, 1, 128)
    CUtensorMap vmap;
    uint16_t* o;         // [B, S, H, 64]
    float* lse;          // [B, H, S]
    const int32_t* len;
    uint32_t* status;
    int B, S, H;
    float scale_log2;
};

// d = max(a, b, c)
__device__ __forceinline__ float max3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (d0, d1) = (a0, a1) * (b0, b1) + (c0, c1), one paired fp32 FMA (round to nearest)
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}

// (d0, d1) += (a0, a1), one paired fp32 add
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1) {
    asm("{\n\t.reg .b64 ra, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rd, {%0, %1};\n\t"
        "add.rn.f32x2 rd, rd, ra;\n\t"
        "mov.b64 {%0, %1}, rd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1));
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The k-th unit of CTA c among G CTAs: snake order over the unit list.
__device__ __forceinline__ int snake_unit(int k, int c, int G) { return k * G + ((k & 1) ? G - 1 - c : c); }

struct Unit {
    int b, h, u, len, nblk;
    bool live_b;         // tile B has a frame inside the clip
};

// Unit t: clip order[r] with cum[r] <= t < cum[r + 1] (r only grows along a
// CTA's walk), frame ranges fastest, heads next.  False past the list.
__device__ __forceinline__ bool unit_at(int t, int& r, const int* slen, const int* order, const int* cum, int B,
                                        Unit& out) {
    while (r < B && cum[r + 1] <= t) ++r;
    if (r >= B) return false;
    const int b = order[r];
    const int len = slen[b];
    const int nt = ceil_div(len, kUnitRows);
    const int v = t - cum[r];
    out.b = b;
    out.h = v / nt;
    out.u = v - out.h * nt;
    out.len = len;
    out.nblk = ceil_div(len, kBN);
    out.live_b = out.u * kUnitRows + kRows < len;
    return true;
}

}  // namespace enc

__global__ void __launch_bounds__(enc::kThreads, 1) encoder_attn_kernel(const __grid_constant__ enc::Params p) {
    using namespace enc;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (smem_u32(smem) & 1023u) {
        if (threadIdx.x == 0) report(p.status, ARK_DEV_TIMEOUT);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + kOffFlag);
    int* slen = reinterpret_cast<int*>(smem + kOffClips);
    int* order = slen + kMaxClips;
    int* cum = order + kMaxClips;
    const int B = p.B, H = p.H, G = gridDim.x, c = blockIdx.x;

    // ---- clip tables: clamped lengths, clips by decreasing block count, unit prefix sums
    if (threadIdx.x < B) {
        int len = __ldg(p.len + threadIdx.x);
        if (len < 0 || len > p.S) {
            if (c == 0) report(p.status, ARK_DEV_BAD_KVLEN);
            len = len < 0 ? 0 : p.S;
        }
        slen[threadIdx.x] = len;
    }
    __syncthreads();
    if (threadIdx.x < B) {
        const int me = threadIdx.x, nb = ceil_div(slen[me], kBN);
        int rank = 0;
        for (int x = 0; x < B; ++x) {
            const int nx = ceil_div(slen[x], kBN);
            rank += (nx > nb || (nx == nb && x < me)) ? 1 : 0;
        }
        order[rank] = me;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        cum[0] = 0;
        for (int r = 0; r < B; ++r) cum[r + 1] = cum[r] + ceil_div(slen[order[r]], kUnitRows) * H;
    }
    __syncthreads();
    const int total = cum[B];
    if (c >= total) return;                                  // no unit for this CTA

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if ((i >= kBarPFull && i < kBarPFull + 2) || (i >= kBarOEmpty && i < kBarOEmpty + 2) ||
                (i >= kBarSRead && i < kBarSRead + 2))
                cnt = kWgThreads;
            mbar_init(&bars[i], cnt);
        }
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
            bool ok = true;
            int r = 0, g = 0;
            int last_q[kQStages] = {-1, -1};        // last unit whose Q went into each buffer
            int last_k[kStages] = {-1, -1, -1};     // last block whose K (V) went into each stage
            int last_v[kStages] = {-1, -1, -1};
            for (int k = 0; ok; ++k) {
                const int t = snake_unit(k, c, G);
                Unit un;
                if (t >= total || !unit_at(t, r, slen, order, cum, B, un)) break;
                const int row0 = un.b * p.S;
                const int qs = k & 1;
                if (k >= kQStages && !(ok = mbar_wait(&bars[kBarQEmpty + qs], ((k >> 1) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[kBarQFull + qs], 2 * kQBytes);
                uint8_t* qd = smem + kOffQ + qs * 2 * kQBytes;
                tma_load_3d(qd, &p.qmap, 0, un.h, row0 + un.u * kUnitRows, &bars[kBarQFull + qs]);
                tma_load_3d(qd + kQBytes, &p.qmap, 0, un.h, row0 + un.u * kUnitRows + kRows, &bars[kBarQFull + qs]);
                last_q[qs] = k;
                for (int j = 0; j < un.nblk; ++j, ++g) {
                    const int st = g % kStages;
                    const uint32_t par = ((g / kStages) - 1) & 1;
                    if (g >= kStages && !(ok = mbar_wait(&bars[kBarKEmpty + st], par))) break;
                    mbar_arrive_expect_tx(&bars[kBarKFull + st], kKV);
                    tma_load_3d(smem + kOffK + st * kKV, &p.kmap, 0, un.h, row0 + j * kBN, &bars[kBarKFull + st]);
                    last_k[st] = g;
                    if (g >= kStages && !(ok = mbar_wait(&bars[kBarVEmpty + st], par))) break;
                    mbar_arrive_expect_tx(&bars[kBarVFull + st], kKV);
                    tma_load_3d(smem + kOffV + st * kKV, &p.vmap, 0, un.h, row0 + j * kBN, &bars[kBarVFull + st]);
                    last_v[st] = g;
                }
            }
            if (!ok) {
                atomicExch(failed_flag, 1);
                report(p.status, ARK_DEV_TIMEOUT);
            }
            // every copy issued has landed before the shared memory can go away (on the normal
            // path the consumers have seen all of them already)
            for (int s = 0; s < kQStages; ++s)
                if (last_q[s] >= 0) (void)mbar_wait(&bars[kBarQFull + s], (last_q[s] >> 1) & 1);
            for (int s = 0; s < kStages; ++s) {
                if (last_k[s] >= 0) (void)mbar_wait(&bars[kBarKFull + s], (last_k[s] / kStages) & 1);
                if (last_v[s] >= 0) (void)mbar_wait(&bars[kBarVFull + s], (last_v[s] / kStages) & 1);
            }
        }
    } else if (warp == 1) {
        // ================================================= score MMAs: S_X = Q_X K^T
        // S_X of the next block is computed as soon as the softmax has read the current one out of
        // tensor memory (P has columns of its own).  Waits are AND-ed over the warp.
        bool ok = true;
        int sx[2] = {0, 0};       // score blocks issued per tile
        int r = 0, g = 0;
        for (int k = 0; ok; ++k) {
            const int t = snake_unit(k, c, G);
            Unit un;
            if (t >= total || !unit_at(t, r, slen, order, cum, B, un)) break;
            const int qs = k & 1;
            const int ntile = un.live_b ? 2 : 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQFull + qs], (k >> 1) & 1)))) break;
            for (int j = 0; j < un.nblk && ok; ++j, ++g) {
                const int st = g % kStages;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarKFull + st], (g / kStages) & 1)))) break;
                for (int x = 0; x < ntile && ok; ++x) {
                    if (sx[x] > 0 &&
                        !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSRead + x], (sx[x] - 1) & 1))))
                        break;
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t qa = sbase + kOffQ + qs * 2 * kQBytes + x * kQBytes;
                        const uint32_t kb = sbase + kOffK + st * kKV;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16(tmem + kColS + x * kBN, umma_desc_sw128(qa + kk * 32, 16, 1024),
                                     umma_desc_sw128(kb + kk * 32, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
                        umma_commit(&bars[kBarSFull + x]);
                    }
                    __syncwarp();
                    ++sx[x];
                }
                if (!ok) break;
                if (lane == 0) {
                    umma_commit(&bars[kBarKEmpty + st]);
                    if (j == un.nblk - 1) umma_commit(&bars[kBarQEmpty + qs]);
                }
                __syncwarp();
            }
        }
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) {
                report(p.status, ARK_DEV_TIMEOUT);
                umma_commit(&bars[kBarDrain]);
                (void)mbar_wait(&bars[kBarDrain], 0);            // MMAs issued so far have completed
            }
            __syncwarp();
        }
    } else if (warp == 10) {
        // ================================================= P V MMAs: O_X += P_X V
        bool ok = true;
        int gx[2] = {0, 0};       // P V blocks issued per tile
        int kx[2] = {0, 0};       // units finished per tile (O_X phases)
        int r = 0, g = 0;
        for (int k = 0; ok; ++k) {
            const int t = snake_unit(k, c, G);
            Unit un;
            if (t >= total || !unit_at(t, r, slen, order, cum, B, un)) break;
            const int ntile = un.live_b ? 2 : 1;
            for (int j = 0; j < un.nblk && ok; ++j, ++g) {
                const int st = g % kStages;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarVFull + st], (g / kStages) & 1)))) break;
                const int live = un.len - j * kBN;           // frames of the clip in this block
                if (live < kBN) {
                    // rows past the clip may hold anything (NaN included): P is 0 there, 0 * NaN is not
                    uint8_t* vt = smem + kOffV + st * kKV;
                    for (int i = lane; i < (kBN - live) * 8; i += 32)
                        *reinterpret_cast<uint4*>(vt + (live + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                    fence_proxy_async_smem();
                }
                __syncwarp();
                const bool last = j == un.nblk - 1;
                for (int x = 0; x < ntile && ok; ++x) {
                    // the first PV of a unit overwrites O_X: the previous unit's epilogue must have read it
                    if (j == 0 && kx[x] > 0 &&
                        !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarOEmpty + x], (kx[x] - 1) & 1))))
                        break;
                    if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPFull + x], gx[x] & 1)))) break;
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t pa = tmem + kColP + x * 64;
                        const uint32_t vb = sbase + kOffV + st * kKV;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk)
                            umma_f16_ts(tmem + kColO + x * kD, pa + kk * 8,
                                        umma_desc_sw128(vb + kk * 16 * 128, kKV, 1024), kIdescPV,
                                        (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&bars[kBarPvDone + x]);
                        if (last) umma_commit(&bars[kBarODone + x]);
                    }
                    __syncwarp();
                    ++gx[x];
                }
                if (!ok) break;
                if (lane == 0) umma_commit(&bars[kBarVEmpty + st]);
                __syncwarp();
            }
            for (int x = 0; x < ntile; ++x) ++kx[x];
        }
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) {
                report(p.status, ARK_DEV_TIMEOUT);
                umma_commit(&bars[kBarDrain + 1]);
                (void)mbar_wait(&bars[kBarDrain + 1], 0);        // MMAs issued so far have completed
            }
            __syncwarp();
        }
    } else {
        // ================================================= softmax + epilogue of tile X
        const int x = (warp - 2) >> 2;                  // 0: tile A (warps 2..5), 1: tile B (warps 6..9)
        const int quad = warp & 3;
        const int rr = quad * 32 + lane;                // this thread's row of the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t col_s = kColS + x * kBN;
        const uint32_t col_o = kColO + x * kD;
        const uint32_t col_p = kColP + x * 64;
        const float sl2 = p.scale_log2;
        bool ok = true;
        int r = 0, gxx = 0, kxx = 0;
        for (int k = 0; ok; ++k) {
            const int t = snake_unit(k, c, G);
            Unit un;
            if (t >= total || !unit_at(t, r, slen, order, cum, B, un)) break;
            if (x == 1 && !un.live_b) continue;          // tile B of this unit has no frame: not computed
            float m_ref = -INFINITY, e0 = 0.f, e1 = 0.f;
            // every tcgen05.ld/st is .sync.aligned and sits on warp-uniform control flow
            for (int j = 0; j < un.nblk; ++j, ++gxx) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + x], gxx & 1));
                if (!ok) break;
                tc_fence_after();
                // two passes over the block's scores, 32 at a time: the row max, then the exponentials;
                // S_X goes back to the score warp once its last chunk has been read again
                const int nvalid = un.len - j * kBN;      // keys of the block inside the clip
                // the last block: keys past the clip get score -inf, hence P = 0
                auto mask32 = [&](uint32_t* w, int k0) {
                    if (nvalid < k0 + 32) {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (k0 + i >= nvalid) w[i] = 0xff800000u;
                    }
                };
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t w[32];
                    tmem_ld32(lane_base + col_s + 32 * c4, w);
                    tmem_wait_ld();
                    mask32(w, 32 * c4);
#pragma unroll
                    for (int i = 0; i < 32; i += 8) {
                        mx[0] = max3(mx[0], __uint_as_float(w[i + 0]), __uint_as_float(w[i + 1]));
                        mx[1] = max3(mx[1], __uint_as_float(w[i + 2]), __uint_as_float(w[i + 3]));
                        mx[2] = max3(mx[2], __uint_as_float(w[i + 4]), __uint_as_float(w[i + 5]));
                        mx[3] = max3(mx[3], __uint_as_float(w[i + 6]), __uint_as_float(w[i + 7]));
                    }
                }
                const float bm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (m_ref == -INFINITY) {
                    m_ref = bm;              // first block: O_X is still empty
                } else if (bm > m_ref + kLazyRescale) {
                    alpha = fast_exp2(m_ref - bm);
                    m_ref = bm;
                    rescale = true;
                }
                const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                // P_X is overwritten below and O_X may be rescaled: the previous PV of the tile must be done
                if (gxx > 0) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone + x], (gxx - 1) & 1));
                    if (!ok) break;
                    tc_fence_after();
                }
                const bool any_rescale = __any_sync(0xffffffffu, rescale);
                if (any_rescale) {
                    e0 *= alpha;
                    e1 *= alpha;
                }
                // P = 2^(s * scale_log2 - mu) as bf16 pairs; 32 keys -> 16 columns of P_X
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    uint32_t w[32];
                    tmem_ld32(lane_base + col_s + 32 * c4, w);
                    tmem_wait_ld();
                    if (c4 == 3) {
                        tc_fence_before();
                        mbar_arrive(&bars[kBarSRead + x]);     // every score of the block has been read
                    }
                    mask32(w, 32 * c4);
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        float x0, x1;
                        fma2(x0, x1, __uint_as_float(w[i]), __uint_as_float(w[i + 1]), sl2, sl2, -mu, -mu);
                        const float s0 = fast_exp2(x0);
                        const float s1 = fast_exp2(x1);
                        add2(e0, e1, s0, s1);
                        pk[i >> 1] = pack_bf16x2(s0, s1);
                    }
                    tmem_st16(lane_base + col_p + 16 * c4, pk);
                }
                if (any_rescale) {
                    // O_X holds the PV of every earlier block (waited for above); rescaled before this
                    // block's P is released to the PV warp, with the scores no longer live
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[16];
                        tmem_ld16(lane_base + col_o + q4 * 16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st16(lane_base + col_o + q4 * 16, o);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[kBarPFull + x]);
            }
            if (!ok) break;
            // ---- epilogue: O_X is complete once every MMA of the unit is
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarODone + x], kxx & 1));
            if (!ok) break;
            tc_fence_after();
            uint32_t oa[64];
            tmem_ld32(lane_base + col_o, *reinterpret_cast<uint32_t(*)[32]>(oa));
            tmem_ld32(lane_base + col_o + 32, *reinterpret_cast<uint32_t(*)[32]>(oa + 32));
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[kBarOEmpty + x]);                    // the next unit may overwrite O_X
            ++kxx;
            const int tt = un.u * kUnitRows + x * kRows + rr;
            if (tt < un.len) {
                const float l = e0 + e1;
                const float inv = 1.f / l;
                uint4* orow = reinterpret_cast<uint4*>(p.o + ((static_cast<size_t>(un.b) * p.S + tt) * H + un.h) * kD);
#pragma unroll
                for (int q8 = 0; q8 < 8; ++q8) {
                    const uint32_t* w = oa + 8 * q8;
                    orow[q8] = make_uint4(pack_bf16x2(__uint_as_float(w[0]) * inv, __uint_as_float(w[1]) * inv),
                                          pack_bf16x2(__uint_as_float(w[2]) * inv, __uint_as_float(w[3]) * inv),
                                          pack_bf16x2(__uint_as_float(w[4]) * inv, __uint_as_float(w[5]) * inv),
                                          pack_bf16x2(__uint_as_float(w[6]) * inv, __uint_as_float(w[7]) * inv));
                }
                p.lse[(static_cast<size_t>(un.b) * H + un.h) * p.S + tt] = (m_ref + __log2f(l)) * kLn2;
            }
        }
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
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

bool enc_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_encoder_mu;       // guards the per-device set-up below (first calls may come from several threads)
bool g_encoder_attr[64];
int g_encoder_sms[64];

}  // namespace

extern "C" ark_status ark_attn_encoder(const void* q, const void* k, const void* v, const int32_t* len, int B, int S,
                                       int H, int D, float scale, void* o, float* lse, uint32_t* d_status,
                                       cudaStream_t stream) {
    if (!q || !k || !v || !len || !o || !lse) return ARK_ERR_INVALID_ARG;
    if (B <= 0 || S <= 0 || H <= 0 || D <= 0 || !(scale > 0.f)) return ARK_ERR_INVALID_ARG;
    if (D != enc::kD || B > enc::kMaxClips) return ARK_ERR_UNSUPPORTED;
    const long long units = (S + enc::kUnitRows - 1) / enc::kUnitRows;
    if (static_cast<long long>(B) * S >= (1LL << 31) || H > 65535 ||
        static_cast<long long>(B) * H * units >= (1LL << 31))
        return ARK_ERR_UNSUPPORTED;
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
    prm.scale_log2 = scale * kLog2e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lk(g_encoder_mu);
        if (!g_encoder_attr[dev]) {
            if (cudaFuncSetAttribute(encoder_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     enc::kSmemBytes) != cudaSuccess)
                return ARK_ERR_CUDA;
            int n = 0;
            if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
                return ARK_ERR_CUDA;
            g_encoder_sms[dev] = n;
            g_encoder_attr[dev] = true;
        }
        sms = g_encoder_sms[dev];
    }
    // persistent: one CTA per SM, at most one per possible unit
    const long long units_max = static_cast<long long>(B) * H * units;
    const int grid = static_cast<int>(units_max < sms ? units_max : sms);
    encoder_attn_kernel<<<grid, enc::kThreads, enc::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}
