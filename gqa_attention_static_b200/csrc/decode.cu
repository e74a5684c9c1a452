// decode.cu -- split-KV single-token GQA decode over a ragged batch, for one
// layer or many independent layers in one launch, with a fused log-sum-exp
// merge of the split partials; and the standalone merge kernel.
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
//   - The work is a list of 16-row K/V tiles: segment (layer l, request b, KV
//     head g) holds ceil(rows/16) tiles, where rows = kv_len[b] (length-aware)
//     or T (masked).  The list is enumerated on the device from kv_len with a
//     prefix sum over the batch in shared memory, so nothing is spent on rows
//     past a request's length.
//   - A persistent grid (a few CTAs per SM) splits the list into one
//     contiguous range of tiles per WARP, equal to within one tile, so every
//     warp streams the same number of bytes whatever the length mix.  A range
//     may start or end inside a segment; that is the split-KV cut.
//   - Each warp streams its range through a private 2-stage ring in shared
//     memory.  One lane issues four TMA tensor loads per tile (K and V, two
//     64-element halves each, 128-byte swizzle so that ldmatrix reads are
//     bank-conflict free); completion is counted on an mbarrier.  The warp
//     keeps streaming across segment boundaries, and the next segment's 8
//     query rows (2 KB) arrive by a bulk copy while the current one runs.
//     The 8 query heads of group g are served from a single read of each K/V
//     row.
//   - Scores are computed transposed, S^T[16 pos x 8 heads] = K_tile * Q^T,
//     with m16n8k16 bf16 tensor-core MMAs: positions fill M = 16 and the 8
//     heads of the group fill N = 8 exactly, so no MMA lane is wasted.  P^T is
//     moved from the accumulator layout to the B-operand layout with two
//     movmatrix transposes, and O^T[dims x heads] += V^T * P^T uses
//     ldmatrix.trans on the same V tile.  fp32 online softmax in the log2
//     domain; per-head maxima across positions by warp shuffles.
//   - A warp that covers a whole segment writes o/lse directly.  A cut
//     segment's pieces write normalised fp32 partials (at most two per warp,
//     with an L2 evict-last hint while the K/V stream is marked evict-first)
//     and the warp moves on: no fence, no counter, no warp ever waits for
//     another.  A second, small kernel (merge_kernel, launched with
//     programmatic dependent launch so that it is resident as soon as decode
//     CTAs retire) recomputes the same partition and merges the pieces of
//     every cut segment by log-sum-exp.
//
// Why tensor cores: per (position, KV head) the kernel reads 512 B and does
// 2 x 8 x 128 multiply-adds, 4 FMA per byte.  At B200 HBM rates that needs
// most of the fp32 FMA pipe; on the tensor pipe it is a few percent.
#include <mutex>

#include "common.cuh"
#include "tma_host.h"

namespace ark {

constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr int kTileRows = 16;
constexpr int kHalfBytes = kTileRows * 128;          // 16 rows x 64 elements, 128B-swizzled
constexpr int kTileBytes = 2 * kHalfBytes;           // one 16-row K or V tile (4 KB)
constexpr int kStageBytes = 2 * kTileBytes;          // K tile + V tile (8 KB)
constexpr int kWarpRing = kStages * kStageBytes;
constexpr int kRingBytes = kWarps * kWarpRing;
constexpr int kQSlotBytes = kGroup * kHeadDim * 2;   // the 8 query rows of one group
constexpr int kQBytes = kWarps * kQSlotBytes;
// fp8 cache: 16-row tiles of 128-byte rows, twice as many stages in the same ring
constexpr int kStages8 = 4;
constexpr int kTileBytes8 = kTileRows * 128;         // one 16-row fp8 K or V tile (2 KB)
constexpr int kStageBytes8 = 2 * kTileBytes8;
static_assert(kStages8 * kStageBytes8 == kWarpRing, "both cache formats use the same ring");
constexpr int kBarBytes = kWarps * (kStages8 + 1) * 8;
constexpr int kMaxBatch = 4096;
constexpr int kMaxWarps = 2048;                      // upper bound on warps per launch (sizes the partials)

struct DecodeCore {
    const int32_t* kv_len;
    uint32_t* status;
    float* part_o;       // [kMaxWarps][2][8][D]  two partial slots per warp
    float* part_lse;     // [kMaxWarps][2][8]
    int L, B, T, Hq, Hkv;
    int min_tiles;       // fewest tiles one warp takes (bounds the pieces per segment)
    int masked;
    float scale_log2;
};

template <int MaxL>
struct DecodeParamsT {
    CUtensorMap kmap[MaxL];   // per layer: cache_k as (128 dims, Hkv, B*T rows), box (64, 1, 16);
    CUtensorMap vmap[MaxL];   // fp8 cache (head-major): (128 bytes, T, B*Hkv), box (128, 16, 1)
    DecodeCore c;
    const uint16_t* q[MaxL];
    uint16_t* o[MaxL];
    float* lse[MaxL];
    const float* k_scale[MaxL];   // fp8 cache only: per layer [Hkv]
    const float* v_scale[MaxL];
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

__device__ __forceinline__ int clamp_len(int x, int T) { return x < 0 ? 0 : (x > T ? T : x); }

// Prefix over the batch of the tiles per request (all KV heads of it):
// s_pref[b] = first tile of request b within a layer, s_pref[B] = tiles per
// layer.  Run by one warp; `report` flags lengths outside [0, T].
__device__ __forceinline__ void tile_prefix(const DecodeCore& c, int* s_pref, int lane, bool report_bad) {
    if (lane == 0) s_pref[0] = 0;
    int run = 0;
    for (int base = 0; base < c.B; base += 32) {
        const int b = base + lane;
        int n = 0;
        if (b < c.B) {
            const int raw = __ldg(c.kv_len + b);
            if ((raw < 0 || raw > c.T) && report_bad) report(c.status, ARK_DEV_BAD_KVLEN);
            const int hi = c.masked ? c.T : clamp_len(raw, c.T);
            n = max(1, (hi + kTileRows - 1) / kTileRows) * c.Hkv;
        }
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, n, off);
            if (lane >= off) n += y;
        }
        if (b < c.B) s_pref[b + 1] = run + n;
        run += __shfl_sync(0xffffffffu, n, 31);
    }
}

// Warps of the decode partition: as many as give every warp at least
// min_tiles tiles, at most the launch's warps.  Warp w takes tiles
// [w N / W, (w + 1) N / W).
__device__ __forceinline__ int partition_warps(const DecodeCore& c, int N, int launch_warps) {
    int W = N / c.min_tiles;
    if (W < 1) W = 1;
    if (W > launch_warps) W = launch_warps;
    return W;
}

template <int MaxL>
struct MergeParamsT {
    DecodeCore c;
    uint16_t* o[MaxL];
    float* lse[MaxL];
    int decode_warps;    // warps of the decode launch whose partials are merged
};

// One segment = (layer, request, KV head): its tiles are s0 .. s0+n-1 of the
// global tile list.  Tile indices fit in 32 bits (the host checks the size).
struct Seg {
    int s0, l, b, g, n, kvl, hi;
};

__device__ __forceinline__ void seg_fill(Seg& s, const int* s_pref, const DecodeCore& c) {
    s.n = (s_pref[s.b + 1] - s_pref[s.b]) / c.Hkv;
    s.kvl = clamp_len(__ldg(c.kv_len + s.b), c.T);
    s.hi = c.masked ? c.T : s.kvl;
}

// Segment of global tile t, and t's index j inside it (binary search over
// the batch prefix; used once per warp).
__device__ __forceinline__ Seg locate(int t, const int* s_pref, int per_layer, const DecodeCore& c, int& j) {
    Seg s;
    s.l = t / per_layer;
    const int r = t - s.l * per_layer;
    int lo = 0, hi = c.B - 1;                // largest b with s_pref[b] <= r
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_pref[mid] <= r) lo = mid; else hi = mid - 1;
    }
    s.b = lo;
    seg_fill(s, s_pref, c);
    const int off = r - s_pref[lo];
    s.g = off / s.n;
    j = off - s.g * s.n;
    s.s0 = t - j;
    return s;
}

// The segment after s in list order: next KV head, then next request, then
// next layer.
__device__ __forceinline__ void seg_next(Seg& s, const int* s_pref, const DecodeCore& c) {
    s.s0 += s.n;
    if (++s.g == c.Hkv) {
        s.g = 0;
        if (++s.b == c.B) {
            s.b = 0;
            ++s.l;
        }
        seg_fill(s, s_pref, c);
    }
}

// Log-sum-exp merge of the pieces of one cut segment (one warp).  Pieces
// come from warps wa..wb; warp wi keeps a piece of this segment in slot 0 if
// the segment began before its range (T0(wi) > s0), in slot 1 otherwise.
// Every lane produces dims 4*lane .. 4*lane+3 of all 8 heads.  Up to
// kFastPieces pieces are read in one round of loads; beyond that, lane i
// first reads the 8 heads' lse of piece wa + i (32 pieces at a time), the
// warp reduces max and sum per head with shuffles, then the pieces' o rows
// are accumulated two pieces per iteration so that 16 loads are in flight.
constexpr int kFastPieces = 3;
__device__ __forceinline__ void merge_pieces(const DecodeCore& c, uint16_t* o, float* lse_out, const Seg& cs, int wa,
                                          int wb, int W, int N, int lane, size_t bh0) {
    const int count = wb - wa + 1;
    auto slot_of = [&](int wi) -> size_t {   // first row of piece wi's 8 heads
        const int sl = (static_cast<long long>(wi) * N >= static_cast<long long>(cs.s0 + 1) * W) ? 0 : 1;
        return (static_cast<size_t>(wi) * 2 + sl) * kGroup;
    };
    if (count <= kFastPieces) {
        // the common case (a segment cut once or twice): every load in one round
        float4 x[kFastPieces][kGroup];
        float lz[kFastPieces][kGroup];
#pragma unroll
        for (int u = 0; u < kFastPieces; ++u) {
            if (u < count) {
                const size_t row = slot_of(wa + u);
                const float4* lsrc = reinterpret_cast<const float4*>(c.part_lse + row);
                const float4 y0 = __ldcg(lsrc), y1 = __ldcg(lsrc + 1);
                lz[u][0] = y0.x; lz[u][1] = y0.y; lz[u][2] = y0.z; lz[u][3] = y0.w;
                lz[u][4] = y1.x; lz[u][5] = y1.y; lz[u][6] = y1.z; lz[u][7] = y1.w;
#pragma unroll
                for (int h = 0; h < kGroup; ++h)
                    x[u][h] = __ldcg(reinterpret_cast<const float4*>(c.part_o + (row + h) * kHeadDim) + lane);
            } else {
#pragma unroll
                for (int h = 0; h < kGroup; ++h) {
                    lz[u][h] = -INFINITY;
                    x[u][h] = make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            float m = lz[0][h];
#pragma unroll
            for (int u = 1; u < kFastPieces; ++u) m = fmaxf(m, lz[u][h]);
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
            float sum = 0.f;
            if (m != -INFINITY) {
#pragma unroll
                for (int u = 0; u < kFastPieces; ++u) {
                    if (lz[u][h] == -INFINITY) continue;   // empty piece: its o is not used
                    const float wgt = fast_exp2((lz[u][h] - m) * kLog2e);
                    sum += wgt;
                    a.x += wgt * x[u][h].x; a.y += wgt * x[u][h].y;
                    a.z += wgt * x[u][h].z; a.w += wgt * x[u][h].w;
                }
            }
            const float iw = (m == -INFINITY) ? 0.f : 1.f / sum;
            uint2 pk;
            pk.x = pack_bf16x2(a.x * iw, a.y * iw);
            pk.y = pack_bf16x2(a.z * iw, a.w * iw);
            reinterpret_cast<uint2*>(o + (bh0 + h) * kHeadDim)[lane] = pk;
            if (lane == 0) lse_out[bh0 + h] = (m == -INFINITY) ? -INFINITY : m + __logf(sum);
        }
        return;
    }
    float M[kGroup], S[kGroup];
#pragma unroll
    for (int h = 0; h < kGroup; ++h) { M[h] = -INFINITY; S[h] = 0.f; }
    auto slot_row = [&](int wi) -> size_t {   // first row of piece wi's 8 heads
        const int sl = (static_cast<long long>(wi) * N >= static_cast<long long>(cs.s0 + 1) * W) ? 0 : 1;
        return (static_cast<size_t>(wi) * 2 + sl) * kGroup;
    };
    for (int base = 0; base < count; base += 32) {
        float l8[kGroup];
        const int i = base + lane;
        if (i < count) {
            const float4* src = reinterpret_cast<const float4*>(c.part_lse + slot_row(wa + i));
            const float4 x0 = __ldcg(src), x1 = __ldcg(src + 1);
            l8[0] = x0.x; l8[1] = x0.y; l8[2] = x0.z; l8[3] = x0.w;
            l8[4] = x1.x; l8[5] = x1.y; l8[6] = x1.z; l8[7] = x1.w;
        } else {
#pragma unroll
            for (int h = 0; h < kGroup; ++h) l8[h] = -INFINITY;
        }
#pragma unroll
        for (int h = 0; h < kGroup; ++h) {
            float m = l8[h];
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
            const float nm = fmaxf(M[h], m);
            float e = (l8[h] == -INFINITY) ? 0.f : fast_exp2((l8[h] - nm) * kLog2e);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) e += __shfl_xor_sync(0xffffffffu, e, off);
            S[h] = (M[h] == -INFINITY ? 0.f : S[h] * fast_exp2((M[h] - nm) * kLog2e)) + e;
            M[h] = nm;
        }
    }
    float4 a[kGroup];
#pragma unroll
    for (int h = 0; h < kGroup; ++h) a[h] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i = 0; i < count; i += 2) {
        float4 x[2][kGroup];
        float l2[2][kGroup];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const bool ok = (i + u) < count;
            const size_t row = slot_row(wa + min(i + u, count - 1));
            const float4* lsrc = reinterpret_cast<const float4*>(c.part_lse + row);
            const float4 y0 = __ldcg(lsrc), y1 = __ldcg(lsrc + 1);
            l2[u][0] = y0.x; l2[u][1] = y0.y; l2[u][2] = y0.z; l2[u][3] = y0.w;
            l2[u][4] = y1.x; l2[u][5] = y1.y; l2[u][6] = y1.z; l2[u][7] = y1.w;
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                x[u][h] = __ldcg(reinterpret_cast<const float4*>(c.part_o + (row + h) * kHeadDim) + lane);
                if (!ok) l2[u][h] = -INFINITY;
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int h = 0; h < kGroup; ++h) {
                if (l2[u][h] == -INFINITY || M[h] == -INFINITY) continue;   // empty piece: never read its o
                const float wgt = fast_exp2((l2[u][h] - M[h]) * kLog2e);
                a[h].x += wgt * x[u][h].x; a[h].y += wgt * x[u][h].y;
                a[h].z += wgt * x[u][h].z; a[h].w += wgt * x[u][h].w;
            }
    }
#pragma unroll
    for (int h = 0; h < kGroup; ++h) {
        const bool emp = (M[h] == -INFINITY);
        const float iw = emp ? 0.f : 1.f / S[h];
        uint2 pk;
        pk.x = pack_bf16x2(a[h].x * iw, a[h].y * iw);
        pk.y = pack_bf16x2(a[h].z * iw, a[h].w * iw);
        reinterpret_cast<uint2*>(o + (bh0 + h) * kHeadDim)[lane] = pk;
        if (lane == 0) lse_out[bh0 + h] = emp ? -INFINITY : M[h] + __logf(S[h]);
    }
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~static_cast<uintptr_t>(1023));
}

// Fp8: the cache holds e4m3 codes (one fp32 scale per layer and KV head for K
// and for V), head-major, so that a tile of 16 positions of one KV head is one
// contiguous 2 KB block (read at 128-byte pieces with a 256-byte stride, as the
// [B,T,Hkv,D] order would give, the same tiles stream about a third slower).
// Tiles are 16 rows of 128 bytes; the MMA fragments are built in
// registers (ld.shared, byte permutes, cvt e4m3x2 -> f16x2, exact) and the MMAs
// run on f16 operands (q converted from bf16 once per segment, P rounded to
// f16).  The head dimension is permuted so that each lane's fragment bytes are
// contiguous: the score dot products are sums over all 128 dims (any common
// order of Q's and K's dims gives the same S), and O's dims are put back in
// place when o is written.
template <int MaxL, bool Fp8>
__global__ void __launch_bounds__(kWarps * 32, 3) decode_kernel(const __grid_constant__ DecodeParamsT<MaxL> p) {
    constexpr int kSt = Fp8 ? kStages8 : kStages;          // ring stages
    constexpr int kStB = Fp8 ? kStageBytes8 : kStageBytes;  // bytes per stage (K tile + V tile)
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    const DecodeCore& c = p.c;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    uint8_t* ring = smem + warp * kWarpRing;
    uint8_t* qslot = smem + kRingBytes + warp * kQSlotBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRingBytes + kQBytes) + warp * (kSt + 1);
    uint64_t* qbar = bars + kSt;
    int* s_pref = reinterpret_cast<int*>(smem + kRingBytes + kQBytes + kBarBytes);   // [B + 1]

    if (lane == 0) {
        for (int s = 0; s <= kSt; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    // q, the cache rows and kv_len may come from the kernel before this one in
    // the stream (the append, or a kernel that advances the lengths): with
    // programmatic dependent launch this grid may be running already, so wait
    // for that grid's completion and its writes before reading any of them (a
    // no-op when there is no such dependency)
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // ---- per CTA: prefix over the batch of the tiles per request (all KV heads)
    if (warp == 0) tile_prefix(c, s_pref, lane, blockIdx.x == 0);
    // the merge grid may be scheduled from here on (it waits for this grid's completion)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    fence_proxy_async_smem();
    __syncthreads();   // the last block-wide barrier: warps run independently from here

    const int per_layer = s_pref[c.B];
    const int N = per_layer * c.L;
    const int W = partition_warps(c, N, static_cast<int>(gridDim.x) * kWarps);
    const int w = blockIdx.x * kWarps + warp;
    if (w >= W) return;
    // warp w takes tiles [T0, T1); tile t belongs to warp floor(((t+1) W - 1) / N)
    const int T0 = static_cast<int>(static_cast<long long>(w) * N / W);
    const int T1 = static_cast<int>(static_cast<long long>(w + 1) * N / W);

    const int lr = lane & 7;
    const int lm = lane >> 3;
    const uint32_t ring_u32 = smem_u32(ring);
    // swizzled ldmatrix addressing: a 16-byte chunk k of row r sits at chunk k ^ (r & 7)
    const uint32_t k_row = (lr + 8 * (lm & 1)) * 128;          // K: matrix lm -> rows 8*(lm&1)
    const uint32_t k_x = (lm >> 1) ^ lr;                       //    and the column chunk lm>>1
    const uint32_t v_row = kTileBytes + (lr + 8 * (lm >> 1)) * 128;   // V^T: rows 8*(lm>>1)
    const uint32_t v_x = (lm & 1) ^ lr;                        //      column chunk lm&1

    // K/V rows are read once per launch; partials are read back by the merge
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    // ---- producer cursor: next tile to issue
    int tp = T0;
    int pj;
    Seg ps = locate(T0, s_pref, per_layer, c, pj);
    uint32_t pseq = 0;
    auto issue_next = [&]() {
        const int st = pseq % kSt;
        if (lane == 0) {
            uint8_t* dst = ring + st * kStB;
            const int row = ps.b * c.T + pj * kTileRows;
            mbar_arrive_expect_tx(&bars[st], kStB);
            if constexpr (Fp8) {
                // head-major cache: the tile is one contiguous 2 KB block of (request, KV head)
                const int hrow = ps.b * c.Hkv + ps.g;
                tma_load_3d_hint(dst, &p.kmap[ps.l], 0, pj * kTileRows, hrow, &bars[st], pol_stream);
                tma_load_3d_hint(dst + kTileBytes8, &p.vmap[ps.l], 0, pj * kTileRows, hrow, &bars[st], pol_stream);
            } else {
                tma_load_3d_hint(dst, &p.kmap[ps.l], 0, ps.g, row, &bars[st], pol_stream);
                tma_load_3d_hint(dst + kHalfBytes, &p.kmap[ps.l], 64, ps.g, row, &bars[st], pol_stream);
                tma_load_3d_hint(dst + kTileBytes, &p.vmap[ps.l], 0, ps.g, row, &bars[st], pol_stream);
                tma_load_3d_hint(dst + kTileBytes + kHalfBytes, &p.vmap[ps.l], 64, ps.g, row, &bars[st],
                                 pol_stream);
            }
        }
        ++pseq;
        ++tp;
        if (++pj == ps.n && tp < T1) {
            seg_next(ps, s_pref, c);
            pj = 0;
        }
    };
    for (int s = 0; s < kSt && tp < T1; ++s) issue_next();

    // ---- query rows of a segment: one 2 KB bulk copy into this warp's slot
    auto issue_q = [&](const Seg& s) {
        if (lane == 0) {
            mbar_arrive_expect_tx(qbar, kQSlotBytes);
            bulk_g2s(qslot, p.q[s.l] + (static_cast<size_t>(s.b) * c.Hq + s.g * kGroup) * kHeadDim, kQSlotBytes,
                     qbar);
        }
    };

    // ---- consumer cursor
    int cj;
    Seg cs = locate(T0, s_pref, per_layer, c, cj);
    issue_q(cs);
    uint32_t qseq = 0;       // query copies consumed
    uint32_t qissued = 1;    // query copies issued
    bool q_next = false;     // the next segment's query rows are still to be fetched
    bool failed = false;
    uint32_t qf[8][2];
    float acc[8][4];
    float m0, m1, e0, e1, r0s, r1s;
    float sl2 = c.scale_log2;   // score scale (log2 domain), times the K scale for an fp8 cache
    float vsc = 1.f;            // V scale of an fp8 cache
    auto begin_segment = [&]() {
        if (!failed && !mbar_wait(qbar, qseq & 1)) {
            failed = true;
            if (lane == 0) report(c.status, ARK_DEV_TIMEOUT);
        }
        ++qseq;
        if constexpr (Fp8) {
            // B fragments of Q^T in f16, head dims permuted: k-step kk of lane (gid, tig) takes
            // dims 32 tig + 4 kk + {0,1} (b0) and + {2,3} (b1) of head gid
            const uint4* qrow = reinterpret_cast<const uint4*>(qslot + gid * 256 + tig * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 x = qrow[i];
                const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xffff0000u);
                    const __half2 h = __floats2half2_rn(lo, hi);
                    qf[2 * i + (j >> 1)][j & 1] = *reinterpret_cast<const uint32_t*>(&h);
                }
            }
            sl2 = c.scale_log2 * __ldg(p.k_scale[cs.l] + cs.g);
            vsc = __ldg(p.v_scale[cs.l] + cs.g);
        } else {
            // B fragments of Q [8 heads][128 dims]: block (heads 0-7, dims 8k..8k+7) -> b0/b1 of k-step k/2
            const uint32_t qa = smem_u32(qslot) + lr * 256 + lm * 16;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                ldsm_x4(qa + i * 64, qf[2 * i][0], qf[2 * i][1], qf[2 * i + 1][0], qf[2 * i + 1][1]);
        }
        __syncwarp();
        // fetch the next segment's rows into the slot once the fragments above
        // have been consumed by the first tile's MMAs
        q_next = (cs.s0 + cs.n < T1);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[mt][i] = 0.f;
        m0 = m1 = -INFINITY;   // running max of heads 2tig, 2tig+1 (log2 domain)
        // this lane's share of the running sums: e* of the fp32 weights (for
        // lse), r* of the bf16-rounded weights that multiply V (to normalise
        // o, so that o stays an exact convex combination of V rows)
        e0 = e1 = r0s = r1s = 0.f;
    };
    begin_segment();

    for (int t = T0; t < T1; ++t) {
        const uint32_t seq = static_cast<uint32_t>(t - T0);
        const int s = seq % kSt;
        if (!failed && !mbar_wait(&bars[s], (seq / kSt) & 1)) {
            failed = true;
            if (lane == 0) report(c.status, ARK_DEV_TIMEOUT);
        }
        if (!failed) {
            const int r0 = cj * kTileRows;
            const uint32_t st = ring_u32 + s * kStB;
            const uint8_t* kt8 = ring + s * kStB;              // fp8: K tile, then the V tile
            const uint8_t* vt8 = kt8 + kTileBytes8;
            const int live = cs.hi - r0;   // rows of this tile that belong to the request's read range
            if (live < kTileRows) {
                // the box also brought rows past the range (next request, or garbage):
                // zero their V rows so that their zero weights never meet a NaN
                const int z0 = max(live, 0);
                if constexpr (Fp8) {
                    uint8_t* vt = ring + s * kStB + kTileBytes8;
                    for (int i = lane; i < (kTileRows - z0) * 8; i += 32)
                        *reinterpret_cast<uint4*>(vt + (z0 + (i >> 3)) * 128 + (i & 7) * 16) = make_uint4(0, 0, 0, 0);
                } else {
                    uint8_t* vt = ring + s * kStB + kTileBytes;
                    for (int i = lane; i < (kTileRows - z0) * 16; i += 32) {
                        const int r = z0 + (i >> 4), part = i & 15;
                        *reinterpret_cast<uint4*>(vt + (part >> 3) * kHalfBytes + r * 128 + (part & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                }
                fence_proxy_async_smem();
            }
            __syncwarp();
            // two independent accumulation chains over the head dim, summed at the end
            float sc[4] = {0.f, 0.f, 0.f, 0.f};
            float sd[4] = {0.f, 0.f, 0.f, 0.f};
            if constexpr (Fp8) {
                // K rows gid and gid+8: bytes (dims) 32 tig .. 32 tig + 31, chunks 2 tig and 2 tig + 1
                // of the 128-byte swizzled rows; word kk holds dims 32 tig + 4 kk .. + 3
                const uint32_t x0 = (2 * tig) ^ (gid & 7), x1 = (2 * tig + 1) ^ (gid & 7);
                const uint4 g0 = *reinterpret_cast<const uint4*>(kt8 + gid * 128 + x0 * 16);
                const uint4 g1 = *reinterpret_cast<const uint4*>(kt8 + gid * 128 + x1 * 16);
                const uint4 h0 = *reinterpret_cast<const uint4*>(kt8 + (gid + 8) * 128 + x0 * 16);
                const uint4 h1 = *reinterpret_cast<const uint4*>(kt8 + (gid + 8) * 128 + x1 * 16);
                const uint32_t wg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
                const uint32_t wh[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a0 = e4m3x2_to_f16x2(static_cast<uint16_t>(wg[kk] & 0xffff));
                    const uint32_t a1 = e4m3x2_to_f16x2(static_cast<uint16_t>(wh[kk] & 0xffff));
                    const uint32_t a2 = e4m3x2_to_f16x2(static_cast<uint16_t>(wg[kk] >> 16));
                    const uint32_t a3 = e4m3x2_to_f16x2(static_cast<uint16_t>(wh[kk] >> 16));
                    mma_f16_16816((kk & 1) ? sd : sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                }
            } else {
#pragma unroll
                for (int kk = 0; kk < 8; kk += 2) {
                    uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                    ldsm_x4(st + (kk >> 2) * kHalfBytes + k_row + (((2 * (kk & 3)) ^ k_x) << 4), a0, a1, a2, a3);
                    ldsm_x4(st + ((kk + 1) >> 2) * kHalfBytes + k_row + (((2 * ((kk + 1) & 3)) ^ k_x) << 4),
                            b0, b1, b2, b3);
                    mma_bf16_16816(sc, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
                    mma_bf16_16816(sd, b0, b1, b2, b3, qf[kk + 1][0], qf[kk + 1][1]);
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) sc[i] += sd[i];
            const bool v0 = (r0 + gid) < cs.kvl;
            const bool v1 = (r0 + gid + 8) < cs.kvl;
            sc[0] = v0 ? sc[0] * sl2 : -INFINITY;
            sc[1] = v0 ? sc[1] * sl2 : -INFINITY;
            sc[2] = v1 ? sc[2] * sl2 : -INFINITY;
            sc[3] = v1 ? sc[3] * sl2 : -INFINITY;

            float t0 = fmaxf(sc[0], sc[2]);
            float t1 = fmaxf(sc[1], sc[3]);
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, o));
                t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, o));
            }
            const float n0 = fmaxf(m0, t0);
            const float n1 = fmaxf(m1, t1);
            const float u0 = (n0 == -INFINITY) ? 0.f : n0;
            const float u1 = (n1 == -INFINITY) ? 0.f : n1;
            // the running max rarely moves once a few tiles are in: skip the rescale then
            const bool moved = __any_sync(0xffffffffu, (n0 != m0) || (n1 != m1));
            const float alpha0 = moved ? fast_exp2(m0 - u0) : 1.f;
            const float alpha1 = moved ? fast_exp2(m1 - u1) : 1.f;
            m0 = n0;
            m1 = n1;

            const float p0 = fast_exp2(sc[0] - u0), p1 = fast_exp2(sc[1] - u1);
            const float p2 = fast_exp2(sc[2] - u0), p3 = fast_exp2(sc[3] - u1);
            // P rounded to the MMA's operand type (bf16, or f16 for an fp8 cache)
            uint32_t p01, p23;
            float q0, q1, q2, q3;   // the rounded weights
            if constexpr (Fp8) {
                const __half2 h01 = __floats2half2_rn(p0, p1), h23 = __floats2half2_rn(p2, p3);
                p01 = *reinterpret_cast<const uint32_t*>(&h01);
                p23 = *reinterpret_cast<const uint32_t*>(&h23);
                q0 = __low2float(h01); q1 = __high2float(h01); q2 = __low2float(h23); q3 = __high2float(h23);
            } else {
                const __nv_bfloat162 b01 = __floats2bfloat162_rn(p0, p1), b23 = __floats2bfloat162_rn(p2, p3);
                p01 = *reinterpret_cast<const uint32_t*>(&b01);
                p23 = *reinterpret_cast<const uint32_t*>(&b23);
                q0 = __low2float(b01); q1 = __high2float(b01); q2 = __low2float(b23); q3 = __high2float(b23);
            }
            e0 = e0 * alpha0 + (p0 + p2);
            e1 = e1 * alpha1 + (p1 + p3);
            r0s = r0s * alpha0 + (q0 + q2);
            r1s = r1s * alpha1 + (q1 + q3);
            if (moved) {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    acc[mt][0] *= alpha0;
                    acc[mt][1] *= alpha1;
                    acc[mt][2] *= alpha0;
                    acc[mt][3] *= alpha1;
                }
            }
            const uint32_t pb0 = movmatrix_t(p01);
            const uint32_t pb1 = movmatrix_t(p23);
            if constexpr (Fp8) {
                // V^T fragments: output dims permuted so that lane gid's rows (gid, gid+8) of
                // block mt are dims 16 gid + 2 mt and 16 gid + 2 mt + 1: one 16-byte chunk
                // (chunk gid) of each of the rows 2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9
                const int ra = 2 * tig;
                const uint4 va = *reinterpret_cast<const uint4*>(vt8 + ra * 128 + ((gid ^ (ra & 7)) << 4));
                const uint4 vb = *reinterpret_cast<const uint4*>(vt8 + (ra + 1) * 128 + ((gid ^ ((ra + 1) & 7)) << 4));
                const uint4 vc = *reinterpret_cast<const uint4*>(vt8 + (ra + 8) * 128 + ((gid ^ (ra & 7)) << 4));
                const uint4 vd = *reinterpret_cast<const uint4*>(vt8 + (ra + 9) * 128 + ((gid ^ ((ra + 1) & 7)) << 4));
                const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
                const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    // bytes 2mt, 2mt+1 of the two rows interleaved: (row a, row b) pairs per dim
                    const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
                    const uint32_t ab = __byte_perm(wa[mt >> 1], wb[mt >> 1], sel);
                    const uint32_t cd = __byte_perm(wc[mt >> 1], wd[mt >> 1], sel);
                    mma_f16_16816(acc[mt], e4m3x2_to_f16x2(static_cast<uint16_t>(ab & 0xffff)),
                                  e4m3x2_to_f16x2(static_cast<uint16_t>(ab >> 16)),
                                  e4m3x2_to_f16x2(static_cast<uint16_t>(cd & 0xffff)),
                                  e4m3x2_to_f16x2(static_cast<uint16_t>(cd >> 16)), pb0, pb1);
                }
            } else {
#pragma unroll
                for (int mt = 0; mt < 8; ++mt) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4_t(st + v_row + (mt >> 2) * kHalfBytes + (((2 * (mt & 3)) ^ v_x) << 4), a0, a1, a2, a3);
                    mma_bf16_16816(acc[mt], a0, a1, a2, a3, pb0, pb1);
                }
            }
            __syncwarp();
            if (tp < T1) issue_next();     // refill the stage just consumed
            if (q_next) {
                Seg nx = cs;
                seg_next(nx, s_pref, c);
                issue_q(nx);
                ++qissued;
                q_next = false;
            }
        }

        if (++cj < cs.n && t + 1 < T1) continue;

        // ---- the consumer leaves segment cs: publish its result
        if (failed) m0 = m1 = -INFINITY;   // a timed-out piece publishes an empty result (lse -inf)
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            e0 += __shfl_xor_sync(0xffffffffu, e0, o);
            e1 += __shfl_xor_sync(0xffffffffu, e1, o);
            r0s += __shfl_xor_sync(0xffffffffu, r0s, o);
            r1s += __shfl_xor_sync(0xffffffffu, r1s, o);
        }
        const bool empty0 = (m0 == -INFINITY), empty1 = (m1 == -INFINITY);
        const float inv0 = empty0 ? 0.f : vsc / r0s;    // vsc = 1 for a bf16 cache
        const float inv1 = empty1 ? 0.f : vsc / r1s;
        const float lse0 = empty0 ? -INFINITY : (m0 + __log2f(e0)) * kLn2;
        const float lse1 = empty1 ? -INFINITY : (m1 + __log2f(e1)) * kLn2;
        const int h0 = 2 * tig, h1 = 2 * tig + 1;
        const size_t bh0 = static_cast<size_t>(cs.b) * c.Hq + cs.g * kGroup;   // row of the group's head 0
        const bool whole = (cs.s0 >= T0) && (cs.s0 + cs.n <= T1);
        if (Fp8 && whole) {
            // lane (gid, tig) holds dims 16 gid .. 16 gid + 15 of heads h0, h1 (the permuted order)
            uint32_t w0[8], w1[8];
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                w0[mt] = pack_bf16x2(acc[mt][0] * inv0, acc[mt][2] * inv0);
                w1[mt] = pack_bf16x2(acc[mt][1] * inv1, acc[mt][3] * inv1);
            }
            uint4* d0 = reinterpret_cast<uint4*>(p.o[cs.l] + (bh0 + h0) * kHeadDim + 16 * gid);
            uint4* d1 = reinterpret_cast<uint4*>(p.o[cs.l] + (bh0 + h1) * kHeadDim + 16 * gid);
            d0[0] = make_uint4(w0[0], w0[1], w0[2], w0[3]);
            d0[1] = make_uint4(w0[4], w0[5], w0[6], w0[7]);
            d1[0] = make_uint4(w1[0], w1[1], w1[2], w1[3]);
            d1[1] = make_uint4(w1[4], w1[5], w1[6], w1[7]);
            if (gid == 0) {
                p.lse[cs.l][bh0 + h0] = lse0;
                p.lse[cs.l][bh0 + h1] = lse1;
            }
        } else if (Fp8) {
            const int slot = (cs.s0 < T0) ? 0 : 1;
            float* po = c.part_o + (static_cast<size_t>(w) * 2 + slot) * kGroup * kHeadDim;
            float* p0r = po + h0 * kHeadDim + 16 * gid;
            float* p1r = po + h1 * kHeadDim + 16 * gid;
#pragma unroll
            for (int mt = 0; mt < 8; mt += 2) {
                st_f32x4_hint(p0r + 2 * mt, acc[mt][0] * inv0, acc[mt][2] * inv0, acc[mt + 1][0] * inv0,
                              acc[mt + 1][2] * inv0, pol_keep);
                st_f32x4_hint(p1r + 2 * mt, acc[mt][1] * inv1, acc[mt][3] * inv1, acc[mt + 1][1] * inv1,
                              acc[mt + 1][3] * inv1, pol_keep);
            }
            if (gid == 0) {
                st_f32_hint(c.part_lse + (static_cast<size_t>(w) * 2 + slot) * kGroup + h0, lse0, pol_keep);
                st_f32_hint(c.part_lse + (static_cast<size_t>(w) * 2 + slot) * kGroup + h1, lse1, pol_keep);
            }
        } else if (whole) {
            __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(p.o[cs.l] + bh0 * kHeadDim);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d = 16 * mt + gid;
                ob[h0 * kHeadDim + d] = __float2bfloat16_rn(acc[mt][0] * inv0);
                ob[h1 * kHeadDim + d] = __float2bfloat16_rn(acc[mt][1] * inv1);
                ob[h0 * kHeadDim + d + 8] = __float2bfloat16_rn(acc[mt][2] * inv0);
                ob[h1 * kHeadDim + d + 8] = __float2bfloat16_rn(acc[mt][3] * inv1);
            }
            if (gid == 0) {
                p.lse[cs.l][bh0 + h0] = lse0;
                p.lse[cs.l][bh0 + h1] = lse1;
            }
        } else {
            const int slot = (cs.s0 < T0) ? 0 : 1;
            float* po = c.part_o + (static_cast<size_t>(w) * 2 + slot) * kGroup * kHeadDim;
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
                const int d = 16 * mt + gid;
                st_f32_hint(po + h0 * kHeadDim + d, acc[mt][0] * inv0, pol_keep);
                st_f32_hint(po + h1 * kHeadDim + d, acc[mt][1] * inv1, pol_keep);
                st_f32_hint(po + h0 * kHeadDim + d + 8, acc[mt][2] * inv0, pol_keep);
                st_f32_hint(po + h1 * kHeadDim + d + 8, acc[mt][3] * inv1, pol_keep);
            }
            if (gid == 0) {
                st_f32_hint(c.part_lse + (static_cast<size_t>(w) * 2 + slot) * kGroup + h0, lse0, pol_keep);
                st_f32_hint(c.part_lse + (static_cast<size_t>(w) * 2 + slot) * kGroup + h1, lse1, pol_keep);
            }
        }
        if (t + 1 < T1) {
            seg_next(cs, s_pref, c);
            cj = 0;
            begin_segment();
        }
    }
    // Never leave with copies in flight: a timed-out warp stops consuming, so
    // wait (bounded) for the tiles and query rows it issued but did not consume.
    // (At most one query copy is in flight at a time, so waiting for the last
    // one issued covers them all; a completed phase returns at once.)
    if (failed) {
        for (uint32_t q2 = pseq > kSt ? pseq - kSt : 0; q2 < pseq; ++q2)
            (void)mbar_wait(&bars[q2 % kSt], (q2 / kSt) & 1);
        (void)mbar_wait(qbar, (qissued - 1) & 1);
    }
}

// One warp per segment (layer, request, KV head): if the decode partition cut
// it, merge its pieces.  Launched right after decode_kernel on the same
// stream, possibly before it has finished (programmatic dependent launch):
// the prefix only reads kv_len; griddepcontrol.wait then blocks until the
// decode grid has completed and its writes are visible.
template <int MaxL>
__global__ void __launch_bounds__(kWarps * 32, 4) merge_kernel(const __grid_constant__ MergeParamsT<MaxL> p) {
    extern __shared__ int s_pref_m[];
    const DecodeCore& c = p.c;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (warp == 0) tile_prefix(c, s_pref_m, lane, false);
    __syncthreads();
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int per_layer = s_pref_m[c.B];
    const int N = per_layer * c.L;
    const int W = partition_warps(c, N, p.decode_warps);
    const int sid = blockIdx.x * kWarps + warp;
    if (sid >= c.L * c.B * c.Hkv) return;
    Seg cs;
    cs.l = sid / (c.B * c.Hkv);
    const int rem = sid - cs.l * c.B * c.Hkv;
    cs.b = rem / c.Hkv;
    cs.g = rem - cs.b * c.Hkv;
    cs.n = (s_pref_m[cs.b + 1] - s_pref_m[cs.b]) / c.Hkv;
    cs.s0 = cs.l * per_layer + s_pref_m[cs.b] + cs.g * cs.n;
    const int wa = static_cast<int>((static_cast<long long>(cs.s0 + 1) * W - 1) / N);
    const int wb = static_cast<int>((static_cast<long long>(cs.s0 + cs.n) * W - 1) / N);
    if (wa == wb) return;                    // one warp covered it and wrote o directly
    const size_t bh0 = static_cast<size_t>(cs.b) * c.Hq + cs.g * kGroup;
    merge_pieces(c, p.o[cs.l], p.lse[cs.l], cs, wa, wb, W, N, lane, bh0);
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

// Fewest 16-row tiles one warp takes: a (request, KV head) of up to
// ceil(T/16) tiles is then cut into at most max_splits + 1 pieces.
int decode_min_tiles(int T, int max_splits) {
    const int tiles = (T + kTileRows - 1) / kTileRows;
    int m = (tiles + max_splits - 1) / max_splits;
    return m < 1 ? 1 : m;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

struct WsLayout {
    size_t part_o, part_lse, total;
};

// Partials of up to kMaxWarps warps, two slots each; nothing in it needs
// initialising and no call leaves state in it for the next.
WsLayout ws_layout() {
    WsLayout w{};
    w.part_o = 0;
    w.part_lse = align256(static_cast<size_t>(kMaxWarps) * 2 * kGroup * kHeadDim * sizeof(float));
    w.total = w.part_lse + align256(static_cast<size_t>(kMaxWarps) * 2 * kGroup * sizeof(float));
    return w;
}

ark_status check_decode_shape(int B, int T, int Hq, int Hkv, int D) {
    if (B <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0) return ARK_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ARK_ERR_INVALID_ARG;
    if (T > ARK_MAX_T) return ARK_ERR_UNSUPPORTED;
    if (D != kHeadDim || Hq / Hkv != kGroup) return ARK_ERR_UNSUPPORTED;
    if (B > kMaxBatch) return ARK_ERR_UNSUPPORTED;
    return ARK_OK;
}

size_t decode_smem(int B) { return 1024 + kRingBytes + kQBytes + kBarBytes + align256((B + 1) * sizeof(int)); }

size_t merge_smem(int B) { return align256((B + 1) * sizeof(int)); }

// SM count and resident CTAs per SM, queried once per device and kernel.
struct DeviceInfo {
    int sms = 0, ctas_per_sm = 0;
};

std::mutex g_device_info_mu;    // guards the per-device tables below (first calls may come from several threads)

template <int MaxL, bool Fp8>
ark_status device_info(DeviceInfo& out) {
    static DeviceInfo table[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_device_info_mu);
    DeviceInfo& d = table[dev];
    if (d.sms == 0) {
        if (cudaFuncSetAttribute(decode_kernel<MaxL, Fp8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(decode_smem(kMaxBatch))) != cudaSuccess)
            return ARK_ERR_CUDA;
        if (cudaFuncSetAttribute(merge_kernel<MaxL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(merge_smem(kMaxBatch))) != cudaSuccess)
            return ARK_ERR_CUDA;
        int sms = 0, per = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return ARK_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, decode_kernel<MaxL, Fp8>, kWarps * 32,
                                                          decode_smem(64)) != cudaSuccess)
            return ARK_ERR_CUDA;
        d.ctas_per_sm = per > 0 ? per : 1;
        d.sms = sms;
    }
    out = d;
    return ARK_OK;
}

// The merge of cut segments: one warp per segment, launched behind the decode
// grid with programmatic stream serialisation (see merge_kernel).
template <int MaxL>
ark_status launch_merge(const DecodeParamsT<MaxL>& prm, int decode_warps, cudaStream_t stream) {
    const DecodeCore& c = prm.c;
    static thread_local MergeParamsT<MaxL> mp;
    mp.c = c;
    for (int l = 0; l < c.L; ++l) {
        mp.o[l] = prm.o[l];
        mp.lse[l] = prm.lse[l];
    }
    mp.decode_warps = decode_warps;
    const long long segs = static_cast<long long>(c.L) * c.B * c.Hkv;
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>((segs + kWarps - 1) / kWarps));
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = merge_smem(c.B);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, merge_kernel<MaxL>, mp) != cudaSuccess) return ARK_ERR_CUDA;
    return ARK_OK;
}

template <int MaxL, bool Fp8>
ark_status launch_decode_core(DecodeParamsT<MaxL>& prm, const void* const* k, const void* const* v, int max_warps,
                              cudaStream_t stream) {
    DecodeCore& c = prm.c;
    for (int l = 0; l < c.L; ++l) {
        const long long rows = static_cast<long long>(c.B) * c.T;
        const bool ok = Fp8 ? (kv8_tensor_map(&prm.kmap[l], k[l], c.B, c.T, c.Hkv, kTileRows) &&
                               kv8_tensor_map(&prm.vmap[l], v[l], c.B, c.T, c.Hkv, kTileRows))
                            : (kv_tensor_map(&prm.kmap[l], k[l], rows, c.Hkv, 64, kTileRows) &&
                               kv_tensor_map(&prm.vmap[l], v[l], rows, c.Hkv, 64, kTileRows));
        if (!ok) return ARK_ERR_CUDA;
    }
    DeviceInfo d;
    ark_status st = device_info<MaxL, Fp8>(d);
    if (st != ARK_OK) return st;
    // tiles in the largest case the device lengths can produce
    const long long max_tiles = static_cast<long long>(c.L) * c.B * c.Hkv * ((c.T + kTileRows - 1) / kTileRows);
    long long grid = static_cast<long long>(d.sms) * d.ctas_per_sm;
    const long long need = (max_tiles / c.min_tiles + kWarps - 1) / kWarps;
    if (need < grid) grid = need;
    if (grid > max_warps / kWarps) grid = max_warps / kWarps;
    if (grid < 1) grid = 1;
    // programmatic stream serialisation: the prologue (prefix over kv_len)
    // overlaps the tail of the previous kernel; see griddepcontrol.wait
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kWarps * 32);
    cfg.dynamicSmemBytes = decode_smem(c.B);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, decode_kernel<MaxL, Fp8>, prm) != cudaSuccess) return ARK_ERR_CUDA;
    return launch_merge<MaxL>(prm, static_cast<int>(grid) * kWarps, stream);
}

template <int MaxL, bool Fp8 = false>
ark_status launch_decode(DecodeParamsT<MaxL>& prm, const void* const* k, const void* const* v, void* workspace,
                         size_t ws_bytes, int max_warps, cudaStream_t stream) {
    DecodeCore& c = prm.c;
    const WsLayout w = ws_layout();
    if (!workspace || ws_bytes < w.total || !aligned16(workspace)) return ARK_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(workspace);
    c.part_o = reinterpret_cast<float*>(base + w.part_o);
    c.part_lse = reinterpret_cast<float*>(base + w.part_lse);
    return launch_decode_core<MaxL, Fp8>(prm, k, v, max_warps, stream);
}

ark_status fill_common(DecodeCore& c, const int32_t* kv_len, int L, int B, int T, int Hq, int Hkv, int D,
                       float scale, ark_decode_mode mode, int max_splits, uint32_t* d_status) {
    if (!kv_len) return ARK_ERR_INVALID_ARG;
    ark_status st = check_decode_shape(B, T, Hq, Hkv, D);
    if (st != ARK_OK) return st;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    if (max_splits <= 0 || !(scale > 0.f) || (mode != ARK_LENGTH_AWARE && mode != ARK_MASKED_STATIC))
        return ARK_ERR_INVALID_ARG;
    const long long max_tiles = static_cast<long long>(L) * B * Hkv * ((T + kTileRows - 1) / kTileRows);
    if (max_tiles >= (1LL << 30)) return ARK_ERR_UNSUPPORTED;
    c.kv_len = kv_len;
    c.status = d_status;
    c.L = L; c.B = B; c.T = T; c.Hq = Hq; c.Hkv = Hkv;
    c.min_tiles = decode_min_tiles(T, max_splits);
    c.masked = (mode == ARK_MASKED_STATIC) ? 1 : 0;
    c.scale_log2 = scale * kLog2e;
    return ARK_OK;
}

}  // namespace

extern "C" size_t ark_attn_decode_layers_workspace_size(int L, int B, int Hq, int D, int T, int max_splits) {
    if (L <= 0 || B <= 0 || Hq <= 0 || D <= 0 || T <= 0 || max_splits <= 0 || Hq % kGroup) return 0;
    return ws_layout().total;
}

extern "C" size_t ark_attn_decode_workspace_size(int B, int Hq, int D, int T, int max_splits) {
    return ark_attn_decode_layers_workspace_size(1, B, Hq, D, T, max_splits);
}

extern "C" ark_status ark_attn_decode(const void* q, const void* cache_k, const void* cache_v,
                                      const int32_t* kv_len, int B, int T, int Hq, int Hkv, int D,
                                      float scale, ark_decode_mode mode, int max_splits,
                                      void* workspace, size_t workspace_bytes,
                                      void* o, float* lse, uint32_t* d_status, cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !o || !lse) return ARK_ERR_INVALID_ARG;
    DecodeParamsT<1> prm{};
    ark_status st = fill_common(prm.c, kv_len, 1, B, T, Hq, Hkv, D, scale, mode, max_splits, d_status);
    if (st != ARK_OK) return st;
    if (!aligned16(q) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return ARK_ERR_INVALID_ARG;
    prm.q[0] = static_cast<const uint16_t*>(q);
    prm.o[0] = static_cast<uint16_t*>(o);
    prm.lse[0] = lse;
    return launch_decode<1>(prm, &cache_k, &cache_v, workspace, workspace_bytes, kMaxWarps, stream);
}

extern "C" ark_status ark_attn_decode_layers(int L, const void* const* q, const void* const* cache_k,
                                             const void* const* cache_v, const int32_t* kv_len, int B, int T,
                                             int Hq, int Hkv, int D, float scale, ark_decode_mode mode,
                                             int max_splits, void* workspace, size_t workspace_bytes,
                                             void* const* o, float* const* lse, uint32_t* d_status,
                                             cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !o || !lse) return ARK_ERR_INVALID_ARG;
    static thread_local DecodeParamsT<ARK_MAX_LAYERS> prm;
    prm = DecodeParamsT<ARK_MAX_LAYERS>{};
    ark_status st = fill_common(prm.c, kv_len, L, B, T, Hq, Hkv, D, scale, mode, max_splits, d_status);
    if (st != ARK_OK) return st;
    for (int l = 0; l < L; ++l) {
        if (!q[l] || !cache_k[l] || !cache_v[l] || !o[l] || !lse[l]) return ARK_ERR_INVALID_ARG;
        if (!aligned16(q[l]) || !aligned16(cache_k[l]) || !aligned16(cache_v[l]) || !aligned16(o[l]) ||
            (reinterpret_cast<uintptr_t>(lse[l]) & 3u))
            return ARK_ERR_INVALID_ARG;
        prm.q[l] = static_cast<const uint16_t*>(q[l]);
        prm.o[l] = static_cast<uint16_t*>(o[l]);
        prm.lse[l] = lse[l];
    }
    return launch_decode<ARK_MAX_LAYERS>(prm, cache_k, cache_v, workspace, workspace_bytes, kMaxWarps, stream);
}

extern "C" ark_status ark_attn_decode_fp8_layers(int L, const void* const* q, const void* const* cache_k,
                                                 const void* const* cache_v, const float* const* k_scale,
                                                 const float* const* v_scale, const int32_t* kv_len, int B, int T,
                                                 int Hq, int Hkv, int D, float scale, ark_decode_mode mode,
                                                 int max_splits, void* workspace, size_t workspace_bytes,
                                                 void* const* o, float* const* lse, uint32_t* d_status,
                                                 cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !k_scale || !v_scale || !o || !lse) return ARK_ERR_INVALID_ARG;
    static thread_local DecodeParamsT<ARK_MAX_LAYERS> prm;
    prm = DecodeParamsT<ARK_MAX_LAYERS>{};
    ark_status st = fill_common(prm.c, kv_len, L, B, T, Hq, Hkv, D, scale, mode, max_splits, d_status);
    if (st != ARK_OK) return st;
    for (int l = 0; l < L; ++l) {
        if (!q[l] || !cache_k[l] || !cache_v[l] || !o[l] || !lse[l] || !k_scale[l] || !v_scale[l])
            return ARK_ERR_INVALID_ARG;
        if (!aligned16(q[l]) || !aligned16(cache_k[l]) || !aligned16(cache_v[l]) || !aligned16(o[l]) ||
            (reinterpret_cast<uintptr_t>(lse[l]) & 3u) || (reinterpret_cast<uintptr_t>(k_scale[l]) & 3u) ||
            (reinterpret_cast<uintptr_t>(v_scale[l]) & 3u))
            return ARK_ERR_INVALID_ARG;
        prm.q[l] = static_cast<const uint16_t*>(q[l]);
        prm.o[l] = static_cast<uint16_t*>(o[l]);
        prm.lse[l] = lse[l];
        prm.k_scale[l] = k_scale[l];
        prm.v_scale[l] = v_scale[l];
    }
    return launch_decode<ARK_MAX_LAYERS, true>(prm, cache_k, cache_v, workspace, workspace_bytes, kMaxWarps, stream);
}

extern "C" ark_status ark_attn_decode_fp8(const void* q, const void* cache_k, const void* cache_v,
                                          const float* k_scale, const float* v_scale, const int32_t* kv_len, int B,
                                          int T, int Hq, int Hkv, int D, float scale, ark_decode_mode mode,
                                          int max_splits, void* workspace, size_t workspace_bytes, void* o,
                                          float* lse, uint32_t* d_status, cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !k_scale || !v_scale || !o || !lse) return ARK_ERR_INVALID_ARG;
    DecodeParamsT<1> prm{};
    ark_status st = fill_common(prm.c, kv_len, 1, B, T, Hq, Hkv, D, scale, mode, max_splits, d_status);
    if (st != ARK_OK) return st;
    if (!aligned16(q) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(k_scale) & 3u) ||
        (reinterpret_cast<uintptr_t>(v_scale) & 3u))
        return ARK_ERR_INVALID_ARG;
    prm.q[0] = static_cast<const uint16_t*>(q);
    prm.o[0] = static_cast<uint16_t*>(o);
    prm.lse[0] = lse;
    prm.k_scale[0] = k_scale;
    prm.v_scale[0] = v_scale;
    return launch_decode<1, true>(prm, &cache_k, &cache_v, workspace, workspace_bytes, kMaxWarps, stream);
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

// ------------------------------------------------ decode without allocation ----
// Scratch of ark_attn_decode_noalloc: partial results for up to
// kNoAllocWarps warps, in one file-scope device array that every GPU
// loading this library holds until the process exits.  Host code must not pass
// the array's name to a kernel (on the host it is a stand-in, not a device
// address); each device's address is looked up once with
// cudaGetSymbolAddress, with that device current.
namespace {

constexpr int kNoAllocWarps = 512;
constexpr size_t kNoAllocPartO = static_cast<size_t>(kNoAllocWarps) * 2 * kGroup * kHeadDim * sizeof(float);
constexpr size_t kNoAllocPartLse = static_cast<size_t>(kNoAllocWarps) * 2 * kGroup * sizeof(float);
constexpr size_t kNoAllocBytes = kNoAllocPartO + kNoAllocPartLse;   // about 4.2 MB

}  // namespace

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocBytes];

namespace {

// The array's address belongs to the module loaded in one CUDA context: after
// a device reset the next context loads the module again, possibly elsewhere.
// So the cached address is keyed by the current context's unique id (driver
// entry points looked up through the runtime; the library links no libcuda).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

std::mutex g_scratch_mu;
void* g_scratch_addr[64];
unsigned long long g_scratch_ctx[64];

bool current_context_id(unsigned long long* id) {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

ark_status scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    // no context may be current yet on this thread's first CUDA call; the symbol
    // lookup below makes the device's primary context current
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    if (!have_ctx || !g_scratch_addr[dev] || g_scratch_ctx[dev] != ctx) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr) return ARK_ERR_CUDA;
        if (!have_ctx && !current_context_id(&ctx)) return ARK_ERR_CUDA;
        g_scratch_addr[dev] = ptr;
        g_scratch_ctx[dev] = ctx;
    }
    *out = g_scratch_addr[dev];
    return ARK_OK;
}

}  // namespace

extern "C" size_t ark_attn_decode_noalloc_scratch_bytes(void) { return kNoAllocBytes; }

extern "C" ark_status ark_attn_decode_noalloc(const void* q, const void* cache_k, const void* cache_v,
                                              const int32_t* kv_len, int B, int T, int Hq, int Hkv, int D,
                                              float scale, ark_decode_mode mode, int max_splits, void* o,
                                              float* lse, uint32_t* d_status, cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !o || !lse) return ARK_ERR_INVALID_ARG;
    DecodeParamsT<1> prm{};
    ark_status st = fill_common(prm.c, kv_len, 1, B, T, Hq, Hkv, D, scale, mode, max_splits, d_status);
    if (st != ARK_OK) return st;
    if (!aligned16(q) || !aligned16(cache_k) || !aligned16(cache_v) || !aligned16(o) ||
        (reinterpret_cast<uintptr_t>(lse) & 3u))
        return ARK_ERR_INVALID_ARG;
    void* base = nullptr;
    if ((st = scratch_address(&base)) != ARK_OK) return st;
    uint8_t* b8 = static_cast<uint8_t*>(base);
    prm.c.part_o = reinterpret_cast<float*>(b8);
    prm.c.part_lse = reinterpret_cast<float*>(b8 + kNoAllocPartO);
    prm.q[0] = static_cast<const uint16_t*>(q);
    prm.o[0] = static_cast<uint16_t*>(o);
    prm.lse[0] = lse;
    return launch_decode_core<1, false>(prm, &cache_k, &cache_v, kNoAllocWarps, stream);
}
