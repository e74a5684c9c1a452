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
// Work: a tile is 128 consecutive frames of one (clip, head); only tiles with
// a frame inside their clip exist.  The kernel is persistent: two CTAs per SM,
// each walking the tile list (clips longest first) in snake order, so that
// the long tiles spread evenly and no CTA is launched for padding.  Inside a
// CTA the tiles run as one pipeline: Q is double-buffered, K and V blocks of
// 64 frames (8 KB each) stream through 4-stage rings, and the first QK^T of
// the next tile is issued before the last PV of the current one.
//
// Per block: S = Q K^T is 4 MMAs of 128x64x16 into a double-buffered TMEM S.
// Warp 0 issues the TMA copies, warp 1 the MMAs (one thread), warps 2..9 run
// the softmax with two threads per row, one for each half of a block's keys.
// The halves are independent: each keeps its own running maximum (lazily
// rescaled), sum and O accumulator in TMEM and stores its P (bf16) over its
// own scores, and O_half += P_half V_half is 2 MMAs of 128x64x16 with P read
// from TMEM and V an MN-major operand.  The two partial results are merged
// once per tile in the epilogue (the rule of a split-KV combine).  Keys past
// len[b] get score -inf (and their V rows are zeroed) in the last block only.
// Rows past len[b] are computed on whatever q holds and are not written.
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
constexpr int kHalfThreads = 128;        // softmax threads of one half (one thread per row)
constexpr int kSoftmaxThreads = 2 * kHalfThreads;
constexpr int kQStages = 2;
constexpr int kStages = 4;               // K and V ring depth
constexpr int kMaxClips = 256;

constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQStages * kQBytes;
constexpr int kOffV = kOffK + kStages * kKV;
constexpr int kOffBar = kOffV + kStages * kKV;
constexpr int kBarQFull = 0;                       // [kQStages]
constexpr int kBarQEmpty = kBarQFull + kQStages;   // [kQStages]: every QK of the tile done
constexpr int kBarKFull = kBarQEmpty + kQStages;   // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages;    // [2]: S buffer
constexpr int kBarPFull = kBarSFull + 2;           // [half][2]: P of a half in TMEM (count 128)
constexpr int kBarPvDone = kBarPFull + 4;          // [half]: PV of a half's keys done (one phase per block)
constexpr int kBarODone = kBarPvDone + 2;          // every MMA of a tile done (one phase per tile)
constexpr int kBarOEmpty = kBarODone + 1;          // O read out by the epilogue (count 256, one phase per tile)
constexpr int kBarDrain = kBarOEmpty + 1;          // MMAs in flight when the MMA warp gives up
constexpr int kBarXchg = kBarDrain + 1;            // [tile parity]: both halves' (max, sum) in shared memory (count 256)
constexpr int kNumBars = kBarXchg + 2;
constexpr int kOffXchg = kOffBar + kNumBars * 8;   // [tile parity][half][max, sum][128] fp32
constexpr int kOffClips = kOffXchg + 2 * 2 * 2 * kRows * 4;
//   int len[kMaxClips] (clamped), order[kMaxClips] (clips, longest first), cum[kMaxClips + 1] (tile prefix)
constexpr int kOffTmemPtr = kOffClips + (3 * kMaxClips + 1) * 4 + 12;
constexpr int kOffFlag = kOffTmemPtr + 8;
constexpr int kSmemBytes = kOffFlag + 16;
static_assert(kOffBar % 8 == 0 && kOffTmemPtr % 8 == 0, "alignment");

// TMEM columns: S buffers 0..63 and 64..127 (fp32 scores; half h's P, bf16
// pairs, over columns 32h..32h+15 of its own scores), O of the keys of half 0
// at 128..191 and of half 1 at 192..255.
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 128;
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

// The k-th tile of CTA c among G CTAs: snake order over the tile list.
__device__ __forceinline__ int snake_tile(int k, int c, int G) { return k * G + ((k & 1) ? G - 1 - c : c); }

// A tile of the list, by the clip tables in shared memory.
struct Tile {
    int b, h, qt, len, nblk;
};

// Tile t: clip order[r] with cum[r] <= t < cum[r + 1] (r only grows along a
// CTA's walk), frames fastest, heads next.  False past the list.
__device__ __forceinline__ bool tile_at(int t, int& r, const int* slen, const int* order, const int* cum, int B,
                                        Tile& out) {
    while (r < B && cum[r + 1] <= t) ++r;
    if (r >= B) return false;
    const int b = order[r];
    const int len = slen[b];
    const int nt = ceil_div(len, kRows);
    const int u = t - cum[r];
    out.b = b;
    out.h = u / nt;
    out.qt = u - out.h * nt;
    out.len = len;
    out.nblk = ceil_div(len, kBN);
    return true;
}

}  // namespace enc

__global__ void __launch_bounds__(enc::kThreads, 2) encoder_attn_kernel(const __grid_constant__ enc::Params p) {
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

    // ---- clip tables: clamped lengths, clips by decreasing block count, tile prefix sums
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
        for (int r = 0; r < B; ++r) cum[r + 1] = cum[r] + ceil_div(slen[order[r]], kRows) * H;
    }
    __syncthreads();
    const int total = cum[B];
    if (c >= total) return;                                  // no tile for this CTA

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if (i >= kBarPFull && i < kBarPFull + 4) cnt = kHalfThreads;
            if (i == kBarOEmpty || i == kBarXchg || i == kBarXchg + 1) cnt = kSoftmaxThreads;
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
            int last_q[kQStages] = {-1, -1};        // last tile whose Q went into each buffer
            int last_k[kStages] = {-1, -1, -1, -1};   // last block whose K (V) went into each stage
            int last_v[kStages] = {-1, -1, -1, -1};
            for (int k = 0; ok; ++k) {
                const int t = snake_tile(k, c, G);
                Tile tl;
                if (t >= total || !tile_at(t, r, slen, order, cum, B, tl)) break;
                const int row0 = tl.b * p.S;
                const int qs = k & 1;
                if (k >= kQStages && !(ok = mbar_wait(&bars[kBarQEmpty + qs], ((k >> 1) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[kBarQFull + qs], kQBytes);
                tma_load_3d(smem + kOffQ + qs * kQBytes, &p.qmap, 0, tl.h, row0 + tl.qt * kRows, &bars[kBarQFull + qs]);
                last_q[qs] = k;
                for (int j = 0; j < tl.nblk; ++j, ++g) {
                    const int st = g % kStages;
                    const uint32_t par = ((g / kStages) - 1) & 1;
                    if (g >= kStages && !(ok = mbar_wait(&bars[kBarKEmpty + st], par))) break;
                    mbar_arrive_expect_tx(&bars[kBarKFull + st], kKV);
                    tma_load_3d(smem + kOffK + st * kKV, &p.kmap, 0, tl.h, row0 + j * kBN, &bars[kBarKFull + st]);
                    last_k[st] = g;
                    if (g >= kStages && !(ok = mbar_wait(&bars[kBarVEmpty + st], par))) break;
                    mbar_arrive_expect_tx(&bars[kBarVFull + st], kKV);
                    tma_load_3d(smem + kOffV + st * kKV, &p.vmap, 0, tl.h, row0 + j * kBN, &bars[kBarVFull + st]);
                    last_v[st] = g;
                }
            }
            if (!ok) {
                atomicExch(failed_flag, 1);
                report(p.status, ARK_DEV_TIMEOUT);
            }
            {
                // every copy issued has landed before the shared memory can go away (on the normal
                // path the consumers have seen all of them already)
                for (int s = 0; s < kQStages; ++s)
                    if (last_q[s] >= 0) (void)mbar_wait(&bars[kBarQFull + s], (last_q[s] >> 1) & 1);
                for (int s = 0; s < kStages; ++s) {
                    if (last_k[s] >= 0) (void)mbar_wait(&bars[kBarKFull + s], (last_k[s] / kStages) & 1);
                    if (last_v[s] >= 0) (void)mbar_wait(&bars[kBarVFull + s], (last_v[s] / kStages) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        bool ok = true;
        // S = Q K^T of block g (block j of tile k)
        auto issue_qk = [&](int k, int j, int g, const Tile& tl) {
            const int qs = k & 1, st = g % kStages;
            if (j == 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQFull + qs], (k >> 1) & 1)))) return;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarKFull + st], (g / kStages) & 1)))) return;
            if (lane == 0) {
                tc_fence_after();
                const uint32_t d = tmem + kColS + (g & 1) * kBN;
                const uint32_t qa = sbase + kOffQ + qs * kQBytes;
                const uint32_t kb = sbase + kOffK + st * kKV;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_f16(d, umma_desc_sw128(qa + kk * 32, 16, 1024), umma_desc_sw128(kb + kk * 32, 16, 1024),
                             kIdescQK, kk > 0 ? 1u : 0u);
                umma_commit(&bars[kBarSFull + (g & 1)]);
                umma_commit(&bars[kBarKEmpty + st]);
                if (j == tl.nblk - 1) umma_commit(&bars[kBarQEmpty + qs]);
            }
            __syncwarp();
        };
        // O_half += P_half V_half for both halves of block g (block j of tile k)
        auto issue_pv = [&](int k, int j, int g, const Tile& tl) {
            const int st = g % kStages;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarVFull + st], (g / kStages) & 1)))) return;
            const int live = tl.len - j * kBN;               // frames of the clip in this block
            if (live < kBN) {
                // rows past the clip may hold anything (NaN included): P is 0 there, 0 * NaN is not
                uint8_t* vt = smem + kOffV + st * kKV;
                for (int i = lane; i < (kBN - live) * 8; i += 32)
                    *reinterpret_cast<uint4*>(vt + (live + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                fence_proxy_async_smem();
            }
            __syncwarp();
            // the first PV of a tile overwrites O: the previous tile's epilogue must have read it
            if (j == 0 && k > 0 && !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarOEmpty], (k - 1) & 1)))) return;
            for (int half = 0; half < 2; ++half) {
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPFull + 2 * half + (g & 1)], (g >> 1) & 1))))
                    return;
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t pa = tmem + kColS + (g & 1) * kBN + half * 32;
                    const uint32_t vb = sbase + kOffV + st * kKV + half * 32 * 128;
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk)
                        umma_f16_ts(tmem + kColO + half * kD, pa + kk * 8,
                                    umma_desc_sw128(vb + kk * 16 * 128, kKV, 1024), kIdescPV,
                                    (j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bars[kBarPvDone + half]);
                }
                __syncwarp();
            }
            if (lane == 0) {
                umma_commit(&bars[kBarVEmpty + st]);
                if (j == tl.nblk - 1) umma_commit(&bars[kBarODone]);
            }
            __syncwarp();
        };
        // walk the blocks of all tiles of this CTA, QK one block ahead of PV
        int r = 0, k = 0, j = 0, g = 0;
        Tile cur, nt;
        bool have = tile_at(snake_tile(0, c, G), r, slen, order, cum, B, cur);
        if (have) issue_qk(0, 0, 0, cur);
        while (have && ok) {
            int nk = k, nj = j + 1;
            bool more = true;
            if (nj == cur.nblk) {
                nk = k + 1;
                nj = 0;
                const int t = snake_tile(nk, c, G);
                more = t < total && tile_at(t, r, slen, order, cum, B, nt);
            } else {
                nt = cur;
            }
            if (more) {
                issue_qk(nk, nj, g + 1, nt);
                if (!ok) break;
            }
            issue_pv(k, j, g, cur);
            if (!ok || !more) break;
            k = nk;
            j = nj;
            cur = nt;
            ++g;
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
    } else {
        // ================================================= softmax + epilogue
        const int quad = warp & 3;
        const int half = (warp - 2) >> 2;               // keys 32*half .. +31 of every block
        const int rr = quad * 32 + lane;                // this thread's row of the tile
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t col_o = kColO + half * kD;
        const float sl2 = p.scale_log2;
        float* xchg = reinterpret_cast<float*>(smem + kOffXchg);
        bool ok = true;
        int r = 0, g = 0;
        for (int k = 0; ok; ++k) {
            const int t = snake_tile(k, c, G);
            Tile tl;
            if (t >= total || !tile_at(t, r, slen, order, cum, B, tl)) break;
            float m_ref = -INFINITY, e0 = 0.f, e1 = 0.f;
            // every tcgen05.ld/st is .sync.aligned and sits on warp-uniform control flow
            for (int j = 0; j < tl.nblk; ++j, ++g) {
                ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + (g & 1)], (g >> 1) & 1));
                if (!ok) break;
                tc_fence_after();
                const uint32_t col_s = kColS + (g & 1) * kBN + half * 32;
                uint32_t v[32];
                tmem_ld32(lane_base + col_s, v);
                tmem_wait_ld();
                const int nvalid = tl.len - j * kBN - half * 32;   // keys of this half inside the clip
                if (nvalid < 32) {
                    // the last block: keys past the clip get score -inf, hence P = 0
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (i >= nvalid) v[i] = 0xff800000u;
                }
                float mx[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t* w = v + 8 * q4;
                    float x = max3(__uint_as_float(w[0]), __uint_as_float(w[1]), __uint_as_float(w[2]));
                    x = max3(x, __uint_as_float(w[3]), __uint_as_float(w[4]));
                    x = max3(x, __uint_as_float(w[5]), __uint_as_float(w[6]));
                    mx[q4] = fmaxf(x, __uint_as_float(w[7]));
                }
                const float bm = fmaxf(max3(mx[0], mx[1], mx[2]), mx[3]) * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (m_ref == -INFINITY) {
                    m_ref = bm;              // first block with a key of this half: O_half is still empty
                } else if (bm > m_ref + kLazyRescale) {
                    alpha = fast_exp2(m_ref - bm);
                    m_ref = bm;
                    rescale = true;
                }
                const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                if (__any_sync(0xffffffffu, rescale)) {
                    // O_half must hold the PV of every earlier block of the tile before it is
                    // rescaled (m_ref was finite before, so j >= 1; PV(g-2) is known complete)
                    ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone + half], (g - 1) & 1));
                    if (!ok) break;
                    tc_fence_after();
                    e0 *= alpha;
                    e1 *= alpha;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint32_t o[16];
                        tmem_ld16(lane_base + col_o + q4 * 16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st16(lane_base + col_o + q4 * 16, o);
                    }
                    tmem_wait_st();
                }
                uint32_t pk[16];
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    float x0, x1;
                    fma2(x0, x1, __uint_as_float(v[i]), __uint_as_float(v[i + 1]), sl2, sl2, -mu, -mu);
                    const float s0 = fast_exp2(x0);
                    const float s1 = fast_exp2(x1);
                    add2(e0, e1, s0, s1);
                    pk[i >> 1] = pack_bf16x2(s0, s1);
                }
                tmem_st16(lane_base + col_s, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[kBarPFull + 2 * half + (g & 1)]);
            }
            if (!ok) break;
            // ---- epilogue: O_0 and O_1 are complete once every MMA of the tile is
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarODone], k & 1));
            if (!ok) break;
            tc_fence_after();
            uint32_t oa[32], ob[32];
            tmem_ld32(lane_base + kColO + half * 32, oa);          // dims 32*half .. +31 from O_0
            tmem_ld32(lane_base + kColO + kD + half * 32, ob);     // and from O_1
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bars[kBarOEmpty]);                        // the next tile may overwrite O
            float* xm = xchg + (k & 1) * 2 * 2 * kRows;             // [half][max, sum][row]
            xm[(half * 2 + 0) * kRows + rr] = m_ref;
            xm[(half * 2 + 1) * kRows + rr] = e0 + e1;
            // a bounded wait (not a named barrier): a softmax warp that gave up never hangs the others
            mbar_arrive(&bars[kBarXchg + (k & 1)]);
            ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarXchg + (k & 1)], (k >> 1) & 1));
            if (!ok) break;
            const float m_oth = xm[((half ^ 1) * 2 + 0) * kRows + rr];
            const float e_oth = xm[((half ^ 1) * 2 + 1) * kRows + rr];
            const int tt = tl.qt * kRows + rr;
            if (tt < tl.len) {
                // O = (2^(m0-M) O_0 + 2^(m1-M) O_1) / (2^(m0-M) l_0 + 2^(m1-M) l_1)
                const float m0 = half == 0 ? m_ref : m_oth, m1 = half == 0 ? m_oth : m_ref;
                const float l0 = half == 0 ? e0 + e1 : e_oth, l1 = half == 0 ? e_oth : e0 + e1;
                const float M = fmaxf(m0, m1);                  // finite for a live row (key 0 is in half 0)
                const float a0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - M);
                const float a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M);
                const float l = l0 * a0 + l1 * a1;
                const float inv = 1.f / l;
                const float c0 = a0 * inv, c1 = a1 * inv;
                uint4* orow = reinterpret_cast<uint4*>(
                    p.o + ((static_cast<size_t>(tl.b) * p.S + tt) * H + tl.h) * kD + half * 32);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    float f[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        f[i] = __uint_as_float(oa[8 * q4 + i]) * c0 + __uint_as_float(ob[8 * q4 + i]) * c1;
                    orow[q4] = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                          pack_bf16x2(f[6], f[7]));
                }
                if (half == 0) p.lse[(static_cast<size_t>(tl.b) * H + tl.h) * p.S + tt] = (M + __log2f(l)) * kLn2;
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

bool g_encoder_attr[64];
int g_encoder_sms[64];

}  // namespace

extern "C" ark_status ark_attn_encoder(const void* q, const void* k, const void* v, const int32_t* len, int B, int S,
                                       int H, int D, float scale, void* o, float* lse, uint32_t* d_status,
                                       cudaStream_t stream) {
    if (!q || !k || !v || !len || !o || !lse) return ARK_ERR_INVALID_ARG;
    if (B <= 0 || S <= 0 || H <= 0 || D <= 0 || !(scale > 0.f)) return ARK_ERR_INVALID_ARG;
    if (D != enc::kD || B > enc::kMaxClips) return ARK_ERR_UNSUPPORTED;
    const long long qt = (S + enc::kRows - 1) / enc::kRows;
    if (static_cast<long long>(B) * S >= (1LL << 31) || H > 65535 ||
        static_cast<long long>(B) * H * qt >= (1LL << 31))
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
    if (!g_encoder_attr[dev]) {
        if (cudaFuncSetAttribute(encoder_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, enc::kSmemBytes) !=
            cudaSuccess)
            return ARK_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return ARK_ERR_CUDA;
        g_encoder_sms[dev] = sms;
        g_encoder_attr[dev] = true;
    }
    // persistent: two CTAs per SM, at most one per possible tile
    const long long tiles_max = static_cast<long long>(B) * H * qt;
    const int grid = static_cast<int>(tiles_max < 2LL * g_encoder_sms[dev] ? tiles_max : 2LL * g_encoder_sms[dev]);
    encoder_attn_kernel<<<grid, enc::kThreads, enc::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}
