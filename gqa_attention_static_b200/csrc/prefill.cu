// prefill.cu -- causal GQA prefill of the prompt on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, operands staged by TMA).
//
// The ONNX model card ("ARK-ASR-3B -- INT8 ONNX", sections Shapes and
// Inference) runs the whole audio+text prompt through the decoder in one call
// ("Prefill, then decode"); each call's key/value rows are written into the
// static cache at cache_position.  Here the rows are already appended (by
// ark_attn_append_rope) and query row t of request b, at absolute position
// p = pos0[b] + t, attends to the cache rows j <= p of its KV head.
//
// Tiling (B200):
//   - One CTA per live tile (16 query positions of request b, KV head g, in
//     one of the launch's layers: up to 16 independent layers per launch).
//     The grid is the upper bound Hkv x B x ceil(S/16) x L; CTA k takes the
//     k-th live tile in order of decreasing absolute position (longest key
//     range first; the layers' copies of a tile next to each other), found on
//     the device from pos0/n_new by a binary search over position levels, so
//     the CTAs that have no tile are the last ones dispatched and never hold a
//     slot ahead of real work, and one launch keeps the SMs busy across
//     layers instead of draining at every layer.  Its 128 MMA
//     rows are the 16 positions x the 8 query heads of group g, so every K/V
//     block is read once for all 8 heads (GQA packing).  The Q tile arrives
//     by two 4-D TMA boxes (64 head-dim elements each, 128-byte swizzle),
//     already in the K-major layout tcgen05 reads.
//   - KV blocks of 64 keys stream in by TMA (3-D boxes over the cache)
//     through 2-stage K and V rings with separate barriers.  S = Q K^T for a block is 8 MMAs of 128x64x16 into a TMEM
//     buffer (two buffers, so QK of block j+1 overlaps the softmax of block
//     j); O += P V is 4 MMAs of 128x128x16 with V as an MN-major operand (no
//     transpose), accumulated in TMEM.  98 KB of shared memory and 256 TMEM
//     columns per CTA: two CTAs share an SM, so one CTA's softmax overlaps the
//     other's loads and MMAs.
//   - Warp roles: warp 0 issues TMA (and owns the TMEM allocation), warp 1
//     issues MMAs from one thread, warps 2..9 run the softmax: two threads
//     per query row (TMEM lane), one for keys 0..31 and one for keys 32..63
//     of each block, which trade their partial row maxima through shared
//     memory behind one named barrier per block.  P (bf16) is stored back to
//     tensor memory over the block's S columns and the PV MMA reads it from
//     there (A operand in TMEM), so shared memory only stages Q, K and V and
//     a K stage is released as soon as its QK MMA has completed.
//   - Softmax in the log2 domain with a lazily moved reference max: O is
//     rescaled (read, scale, write back in TMEM) only when a row's block max
//     exceeds its reference by more than 2^8, which for real data is almost
//     never after the first block.  Rows past n_new[b] are computed on
//     whatever the padded q holds and never written.
//   - Only the last block needs the causal mask; V rows past the causal range
//     of the tile are zeroed in shared memory before their (zero-weight) use,
//     so garbage past the valid rows cannot turn into NaN.
//
// Roofline: per request of L prompt rows and per layer, 4096 * L * (L + 1)
// FLOPs (the causal half of QK^T and PV for 16 heads) against 9216 * L bytes
// (q read, o written, K/V rows read once per tile from L2); at the prompt
// lengths of the coalesced-prefill workload (<= 387) that is HBM- and
// latency-bound rather than tensor-bound.
#include "common.cuh"
#include "tma_host.h"

#include <mutex>

namespace ark {
namespace pf {

constexpr int kRows = 128;               // MMA M: 16 positions x 8 heads
constexpr int kPos = 16;                 // query positions per tile
constexpr int kBN = 64;                  // keys per KV block
constexpr int kQHalf = kRows * 128;      // one 64-element half of the Q tile (16 KB)
constexpr int kKHalf = kBN * 128;        // one 64-element half of a K or V block (8 KB)
constexpr int kKV = 2 * kKHalf;          // a K or V block (16 KB); also holds P (128 rows x 64 keys)
constexpr int kThreads = 320;            // warp 0: TMA, warp 1: MMA, warps 2..9: softmax
constexpr int kSoftmaxThreads = 256;     // two threads per row: keys 0..31 and 32..63 of a block

constexpr int kKStages = 2;
constexpr int kVStages = 2;

// shared memory map (the dynamic shared memory base is 1024-aligned)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + 2 * kQHalf;          // kKStages stages
constexpr int kOffV = kOffK + kKStages * kKV;      // kVStages stages
constexpr int kOffBar = kOffV + kVStages * kKV;
constexpr int kBarQ = 0;
constexpr int kBarKFull = 1;                       // kKStages
constexpr int kBarKEmpty = kBarKFull + kKStages;   // kKStages
constexpr int kBarVFull = kBarKEmpty + kKStages;   // kVStages
constexpr int kBarVEmpty = kBarVFull + kVStages;   // kVStages
constexpr int kBarSFull = kBarVEmpty + kVStages;   // 2
constexpr int kBarPFull = kBarSFull + 2;           // 2
constexpr int kBarPvDone = kBarPFull + 2;
constexpr int kBarQRot = kBarPvDone + 1;           // rotated Q tile in place (count: softmax threads)
constexpr int kBarODone = kBarQRot + 1;            // every MMA of the tile done (one phase)
constexpr int kNumBars = kBarODone + 1;
constexpr int kOffXchg = kOffBar + kNumBars * 8;   // [3][2 halves][128 rows] fp32: row max (by block
                                                   // parity) and row sum exchange between a row's two threads
constexpr int kOffTmemPtr = kOffXchg + 3 * 2 * kRows * 4;
constexpr int kOffFlag = kOffTmemPtr + 8;
constexpr int kSmemBytes = kOffFlag + 16;

// TMEM columns
constexpr uint32_t kColS = 0;            // two S buffers: 0..63, 64..127
constexpr uint32_t kColO = 128;          // O: 128..255
constexpr uint32_t kTmemCols = 256;

// instruction descriptors (kind::f16): D fp32, A/B bf16, M = 128
constexpr uint32_t kIdescF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);
constexpr uint32_t kIdescQK = kIdescF16 | ((64u >> 3) << 17);                // N = 64 keys, B = K (K-major)
constexpr uint32_t kIdescPV = kIdescF16 | ((128u >> 3) << 17) | (1u << 16);  // N = 128 dims, B = V (MN-major)

constexpr float kLazyRescale = 8.0f;     // log2 units: rescale O only past a factor 2^8

// layers per launch: four tensor maps per layer in the kernel parameters
// (which hold at most 32 KB)
constexpr int kLayersPerLaunch = 16;

struct Params {
    CUtensorMap qmap[kLayersPerLaunch];   // q as (128, 8, Hq/8, B*S), box (64, 8, 1, 16)
    CUtensorMap kmap[kLayersPerLaunch];   // cache_k as (128, Hkv, B*T), box (64, 1, 64)
    CUtensorMap vmap[kLayersPerLaunch];
    CUtensorMap omap[kLayersPerLaunch];   // o as q, box (64, 8, 1, 1): one position, 8 heads, 64 dims
    float* lse[kLayersPerLaunch];         // [B, Hq, S]
    const int32_t* pos0;
    const int32_t* n_new;
    uint32_t* status;
    const float4* table;                  // rotary table [T][64] {cos, sin} (fp32), for the fused-RoPE form
    int B, S, T, Hq, Hkv, L;
    float scale_log2;
};

}  // namespace pf

// Named barrier 1 over the 256 softmax threads, returning the AND of `pred`
// over all of them (so that decisions taken after it are the same everywhere).
__device__ __forceinline__ bool bar_and_all(bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, 1, %2, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(out) : "r"(static_cast<uint32_t>(pred)), "n"(pf::kSoftmaxThreads) : "memory");
    return out != 0;
}

namespace pf {

// Request b's lengths as the kernel uses them (device values, clamped into
// range; `bad` when they had to be), and its tiles' position levels: tile qt
// of request b sits at level (pos0 >> 4) + qt, and the request has
// ceil(n_new / 16) tiles.
struct ReqTiles {
    int nn, p0, lev0, ntiles;
    bool bad;
};

__device__ __forceinline__ ReqTiles req_tiles(const Params& p, int b) {
    ReqTiles t;
    int nn = __ldg(p.n_new + b);
    int p0 = __ldg(p.pos0 + b);
    t.bad = nn < 0 || nn > p.S || p0 < 0 || p0 + (nn < 0 ? 0 : (nn > p.S ? p.S : nn)) > p.T;
    if (t.bad) {
        nn = nn < 0 ? 0 : (nn > p.S ? p.S : nn);
        if (p0 < 0) p0 = 0;
        if (p0 > p.T) p0 = p.T;
        if (p0 + nn > p.T) nn = p.T - p0;
    }
    t.nn = nn;
    t.p0 = p0;
    t.lev0 = p0 >> 4;
    t.ntiles = (nn + kPos - 1) / kPos;
    return t;
}

// tiles of a request at levels >= lam
__device__ __forceinline__ int tiles_at_or_above(const ReqTiles& t, int lam) {
    const int c = t.lev0 + t.ntiles - max(lam, t.lev0);
    return c < 0 ? 0 : c;
}

// The j-th live tile in the order (level descending, request ascending),
// computed by one warp (every lane returns the same result).  Lane l handles
// requests l, l + 32, ...; C(lam) = tiles at levels >= lam is non-increasing,
// and the tile's level is the largest lam with C(lam) > j.
struct TilePick {
    int b, qt, nn, p0;
    bool live;
};

__device__ __forceinline__ TilePick pick_tile(const Params& p, int j, int lane, bool report_bad) {
    const unsigned full = 0xffffffffu;
    ReqTiles mine{0, 0, 0, 0, false};
    if (lane < p.B) mine = req_tiles(p, lane);
    bool bad = mine.bad;
    auto count = [&](int lam) {
        int c = lane < p.B ? tiles_at_or_above(mine, lam) : 0;
        for (int bb = 32 + lane; bb < p.B; bb += 32) {
            const ReqTiles t = req_tiles(p, bb);
            c += tiles_at_or_above(t, lam);
            bad |= t.bad;
        }
        return static_cast<int>(__reduce_add_sync(full, static_cast<unsigned>(c)));
    };
    TilePick r{0, 0, 0, 0, false};
    const int total = count(0);
    if (report_bad && __any_sync(full, bad) && lane == 0) report(p.status, ARK_DEV_BAD_POS);
    if (j >= total) return r;
    int lo = 0, hi = (p.T + kPos - 1) / kPos;     // C(lo) > j, C(hi) == 0
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (count(mid) > j) lo = mid;
        else hi = mid;
    }
    int rank = j - count(lo + 1);                 // among the tiles at level lo, by request
    for (int base = 0; base < p.B; base += 32) {
        const ReqTiles t = base == 0 ? mine : (base + lane < p.B ? req_tiles(p, base + lane) : ReqTiles{0, 0, 0, 0, false});
        const bool at = base + lane < p.B && t.lev0 <= lo && lo < t.lev0 + t.ntiles;
        const unsigned m = __ballot_sync(full, at);
        const int n = __popc(m);
        if (rank < n) {
            const int src = static_cast<int>(__fns(m, 0, rank + 1));
            r.b = base + src;
            r.nn = __shfl_sync(full, t.nn, src);
            r.p0 = __shfl_sync(full, t.p0, src);
            r.qt = lo - __shfl_sync(full, t.lev0, src);
            r.live = true;
            return r;
        }
        rank -= n;
    }
    return r;                                     // not reached for consistent counts
}

}  // namespace pf

// Rope: q arrives unrotated and the softmax warps rotate the Q tile in shared
// memory (Qwen2 rotate-half at the row's absolute position, the products in
// double from the bf16 input and the fp32 table, one rounding to bf16: the
// same values ark_attn_append_rope writes), before the first QK MMA.
template <bool Rope>
__global__ void __launch_bounds__(pf::kThreads, 2) prefill_kernel(const __grid_constant__ pf::Params p) {
    using namespace pf;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = blockIdx.x % p.Hkv;
    if (smem_u32(smem) & 1023u) {                           // the swizzled layouts need 1024-byte alignment
        if (threadIdx.x == 0) report(p.status, ARK_DEV_TIMEOUT);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + kOffFlag);

    // barrier init and the TMEM allocation overlap the tile search's loads
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i)
            mbar_init(&bars[i], (i == kBarPFull || i == kBarPFull + 1 || i == kBarQRot) ? kSoftmaxThreads : 1);
        *failed_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_ptr, kTmemCols);
    // every warp finds the CTA's tile by itself (same inputs, same result);
    // consecutive CTAs take the same tile of consecutive layers
    const int lt = static_cast<int>(blockIdx.x / p.Hkv);
    const int l = lt % p.L;
    const TilePick tile = pick_tile(p, lt / p.L, lane, blockIdx.x == 0 && warp == 0);
    const int b = tile.b, qt = tile.qt, nn = tile.nn, p0 = tile.p0;
    const int t0 = qt * kPos;
    const int kv_end = p0 + min(t0 + kPos, nn);             // keys visible to the tile's last row
    const int nblk = tile.live ? (kv_end + kBN - 1) / kBN : 0;

    auto load_k = [&](int j) {
        const int ks = j % kKStages;
        mbar_arrive_expect_tx(&bars[kBarKFull + ks], kKV);
        uint8_t* kd = smem + kOffK + ks * kKV;
        tma_load_3d(kd, &p.kmap[l], 0, g, b * p.T + j * kBN, &bars[kBarKFull + ks]);
        tma_load_3d(kd + kKHalf, &p.kmap[l], 64, g, b * p.T + j * kBN, &bars[kBarKFull + ks]);
    };
    auto load_v = [&](int j) {
        const int vs = j % kVStages;
        mbar_arrive_expect_tx(&bars[kBarVFull + vs], kKV);
        uint8_t* vd = smem + kOffV + vs * kKV;
        tma_load_3d(vd, &p.vmap[l], 0, g, b * p.T + j * kBN, &bars[kBarVFull + vs]);
        tma_load_3d(vd + kKHalf, &p.vmap[l], 64, g, b * p.T + j * kBN, &bars[kBarVFull + vs]);
    };
    // the first blocks need no free stage: thread 0 (which initialised the
    // barriers) issues them before the CTA barrier
    constexpr int kPre = 2;
    static_assert(kKStages >= kPre && kVStages >= kPre, "preloaded blocks need their own stages");
    if (threadIdx.x == 0 && tile.live) {
        mbar_arrive_expect_tx(&bars[kBarQ], 2 * kQHalf);
        const int qrow = b * p.S + t0;
        tma_load_4d(smem + kOffQ, &p.qmap[l], 0, 0, g, qrow, &bars[kBarQ]);
        tma_load_4d(smem + kOffQ + kQHalf, &p.qmap[l], 64, 0, g, qrow, &bars[kBarQ]);
        for (int j = 0; j < min(nblk, kPre); ++j) {
            load_k(j);
            load_v(j);
        }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    if (!tile.live) {                                       // whole CTA: no live tile
        if (warp == 0) tmem_dealloc(tmem, kTmemCols);
        return;
    }
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            bool ok = true;
            for (int j = kPre; j < nblk; ++j) {
                // K stage is free once the QK MMA of block j - kKStages is done
                if (!mbar_wait(&bars[kBarKEmpty + j % kKStages], ((j / kKStages) - 1) & 1)) {
                    ok = false;
                    break;
                }
                load_k(j);
                // V stage is free once PV of block j - kVStages is done
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
        // waits are AND-ed over the warp so that the __syncwarp()s below are reached by all lanes
        bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[Rope ? kBarQRot : kBarQ], 0));
        auto wait_k = [&](int j) {
            return __all_sync(0xffffffffu, mbar_wait(&bars[kBarKFull + j % kKStages], (j / kKStages) & 1));
        };
        auto wait_v = [&](int j) {
            // V block j landed; zero its rows past the tile's causal range
            if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarVFull + j % kVStages], (j / kVStages) & 1)))
                return false;
            const int live = kv_end - j * kBN;
            if (live < kBN) {
                uint8_t* vt = smem + kOffV + (j % kVStages) * kKV;
                for (int i = lane; i < (kBN - live) * 16; i += 32) {
                    const int r = live + (i >> 4), part = i & 15;
                    *reinterpret_cast<uint4*>(vt + (part >> 3) * kKHalf + r * 128 + (part & 7) * 16) =
                        make_uint4(0, 0, 0, 0);
                }
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
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t sub = (kk & 3) * 32;
                    umma_f16(d, umma_desc_sw128(sbase + kOffQ + (kk >> 2) * kQHalf + sub, 16, 1024),
                             umma_desc_sw128(kb + (kk >> 2) * kKHalf + sub, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bars[kBarSFull + (j & 1)]);
                umma_commit(&bars[kBarKEmpty + j % kKStages]);
            }
            __syncwarp();
        };
        auto issue_pv = [&](int j) {
            if (lane == 0) {
                tc_fence_after();
                // P of block j: bf16 pairs in the first 32 columns of its S buffer
                const uint32_t pa = tmem + kColS + (j & 1) * kBN;
                const uint32_t vb = sbase + kOffV + (j % kVStages) * kKV;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    umma_f16_ts(tmem + kColO, pa + kk * 8, umma_desc_sw128(vb + kk * 16 * 128, kKHalf, 1024),
                                kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&bars[kBarVEmpty + j % kVStages]);
                umma_commit(&bars[kBarPvDone]);
            }
            __syncwarp();
        };
        if (ok) ok = wait_k(0);
        if (ok) issue_qk(0);
        for (int j = 0; j < nblk && ok; ++j) {
            if (j + 1 < nblk) {
                // S buffer (j+1)&1 was last read by the softmax of block j-1 (its P arrival was waited below)
                if (!(ok = wait_k(j + 1))) break;
                issue_qk(j + 1);
            }
            // P of block j is in TMEM (and S buffer j&1 is not reused before PV(j): MMAs run in issue order)
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPFull + (j & 1)], (j >> 1) & 1)))) break;
            if (!(ok = wait_v(j))) break;
            issue_pv(j);
        }
        if (ok && lane == 0) umma_commit(&bars[kBarODone]);
        __syncwarp();
        if (!ok && lane == 0) {
            atomicExch(failed_flag, 1);
            report(p.status, ARK_DEV_TIMEOUT);
        }
    } else {
        // ================================================= softmax + epilogue
        const int quad = warp & 3;                      // TMEM lanes 32*quad .. +31
        const int half = (warp - 2) >> 2;               // 0: keys 0..31 of a block, 1: keys 32..63
        const int r = quad * 32 + lane;                 // this thread's row of the tile
        const int tr = t0 + (r >> 3);                   // its query position (within the call)
        const int hh = r & 7;
        const int prow = p0 + tr;                       // its absolute position
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        float* xchg = reinterpret_cast<float*>(smem + kOffXchg);   // [half][row]
        float m_ref = -INFINITY, e_sum = 0.f, r_sum = 0.f;         // this half's share of the row sums
        bool ok = true;
        if constexpr (Rope) {
            // rotate the Q tile in place: item = (row, 16-byte chunk); the chunk holds dims 8c..8c+7
            // in the first half and their rotary partners 64 + 8c.. in the second, at the same offset
            ok = mbar_wait(&bars[kBarQ], 0);
            if (ok) {
                for (int it = threadIdx.x - 64; it < kRows * 8; it += kSoftmaxThreads) {
                    const int rr = it >> 3, cch = it & 7;
                    if (t0 + (rr >> 3) >= nn) continue;                 // padded rows are never stored
                    const int pos = p0 + t0 + (rr >> 3);
                    const uint32_t off = rr * 128 + ((cch ^ (rr & 7)) << 4);
                    uint4* plo = reinterpret_cast<uint4*>(smem + kOffQ + off);
                    uint4* phi = reinterpret_cast<uint4*>(smem + kOffQ + kQHalf + off);
                    const uint4 xlo = *plo, xhi = *phi;
                    const uint32_t wl[4] = {xlo.x, xlo.y, xlo.z, xlo.w}, wh[4] = {xhi.x, xhi.y, xhi.z, xhi.w};
                    uint32_t ol[4], oh[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float4 cs = __ldg(p.table + static_cast<size_t>(pos) * 32 + 4 * cch + j);  // pairs 2j, 2j+1
                        const double c0 = cs.x, s0 = cs.y, c1 = cs.z, s1 = cs.w;
                        const double a0 = bf16_bits_to_f64(static_cast<uint16_t>(wl[j] & 0xffff));
                        const double a1 = bf16_bits_to_f64(static_cast<uint16_t>(wl[j] >> 16));
                        const double h0 = bf16_bits_to_f64(static_cast<uint16_t>(wh[j] & 0xffff));
                        const double h1 = bf16_bits_to_f64(static_cast<uint16_t>(wh[j] >> 16));
                        // both products are exact in double, so contraction cannot change the result
                        ol[j] = static_cast<uint32_t>(f64_to_bf16_rn(a0 * c0 - h0 * s0)) |
                                (static_cast<uint32_t>(f64_to_bf16_rn(a1 * c1 - h1 * s1)) << 16);
                        oh[j] = static_cast<uint32_t>(f64_to_bf16_rn(h0 * c0 + a0 * s0)) |
                                (static_cast<uint32_t>(f64_to_bf16_rn(h1 * c1 + a1 * s1)) << 16);
                    }
                    *plo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                    *phi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                }
            }
            fence_proxy_async_smem();                          // the MMA reads the tile through the async proxy
            mbar_arrive(&bars[kBarQRot]);
        }
        // Every tcgen05.ld/st below is .sync.aligned: all 32 lanes of the warp
        // execute it together, so all control flow around them is warp-uniform;
        // the loop itself is left by all 256 softmax threads together (its exit
        // test is AND-reduced by the named barrier), so barrier 1 never deadlocks.
        for (int j = 0; j < nblk; ++j) {
            ok = __all_sync(0xffffffffu, ok && mbar_wait(&bars[kBarSFull + (j & 1)], (j >> 1) & 1));
            tc_fence_after();
            const uint32_t scol = lane_base + kColS + (j & 1) * kBN + half * 32;
            const int nvalid = min(32, prow - j * kBN - half * 32 + 1);   // visible keys of this half
            uint32_t v[32];
            tmem_ld32(scol, v);
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
            // trade partial maxima with the other half of the row (buffer chosen by block parity)
            float* xm = xchg + (j & 1) * 2 * kRows;
            xm[half * kRows + r] = my_max;
            if (!bar_and_all(ok)) {
                ok = false;
                break;
            }
            const float bm = fmaxf(my_max, xm[(half ^ 1) * kRows + r]) * p.scale_log2;
            float alpha = 1.f;
            bool rescale = false;
            if (m_ref == -INFINITY) {
                m_ref = bm;                 // first visible block of this row: O is still empty
            } else if (bm > m_ref + kLazyRescale) {
                alpha = fast_exp2(m_ref - bm);
                m_ref = bm;
                rescale = true;
            }
            const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
            if (__any_sync(0xffffffffu, rescale)) {
                // O must hold PV of every earlier block before it is rescaled
                if (j >= 1) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone], (j - 1) & 1));
                tc_fence_after();
                e_sum *= alpha;
                r_sum *= alpha;
#pragma unroll
                for (int c = 0; c < 4; ++c) {         // this half rescales O columns 64*half .. +63
                    uint32_t o[16];
                    tmem_ld16(lane_base + kColO + half * 64 + c * 16, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                    tmem_st16(lane_base + kColO + half * 64 + c * 16, o);
                }
                tmem_wait_st();
            }
            // P = exp2(s * scale_log2 - m_ref) as bf16 pairs, stored over the block's S columns:
            // keys 2c, 2c+1 in column c, this half's keys 32*half .. +31 in columns 16*half .. +15
            // (both halves finished reading S before the barrier above)
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
        // O is complete once every MMA of the tile is (a barrier of its own: the per-block one
        // may still be a phase short of PV(nblk-2) here, and its parity would not tell)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarODone], 0));
        tc_fence_after();
        // the row sums of both halves (every softmax thread reaches these barriers)
        float* xs = xchg + 2 * 2 * kRows;
        xs[half * kRows + r] = e_sum;
        ok = bar_and_all(ok);
        const float e_tot = e_sum + xs[(half ^ 1) * kRows + r];
        ok = bar_and_all(ok);
        xs[half * kRows + r] = r_sum;
        ok = bar_and_all(ok);
        const float r_tot = r_sum + xs[(half ^ 1) * kRows + r];
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        } else {
            // epilogue: o row = O / sum of the bf16 weights; lse from the fp32 weights.
            // This half's 64 dims of the row go, as bf16, to the (finished) Q tile in shared
            // memory, in the 128-byte-swizzled layout of a (64, 8 heads) TMA box per position;
            // each warp then stores its 4 positions (its 32 rows) with TMA, live positions only.
            const bool live = tr < nn;
            const float inv = 1.f / r_tot;
            const int h = g * kGroup + hh;
            uint8_t* stage = smem + kOffQ + half * kQHalf + r * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[16];
                tmem_ld16(lane_base + kColO + half * 64 + c * 16, o);
                tmem_wait_ld();
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
                    *reinterpret_cast<uint4*>(stage + (((2 * c + q) ^ (r & 7)) << 4)) = w;
                }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane < 4) {
                const int pp = quad * 4 + lane;              // position of the tile
                if (t0 + pp < nn) {
                    tma_store_4d(&p.omap[l], smem + kOffQ + half * kQHalf + pp * 1024, half * 64, 0, g,
                                 b * p.S + t0 + pp);
                    bulk_commit();
                    bulk_wait_read();
                }
            }
            if (live && half == 0)
                p.lse[l][(static_cast<size_t>(b) * p.Hq + h) * p.S + tr] = (m_ref + __log2f(e_tot)) * kLn2;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        if (*failed_flag) {
            // do not release shared or tensor memory under copies or MMAs still in flight
            for (int s = 0; s < kKStages; ++s) (void)mbar_wait(&bars[kBarKFull + s], 0);
            for (int s = 0; s < kVStages; ++s) (void)mbar_wait(&bars[kBarVFull + s], 0);
            (void)mbar_wait(&bars[kBarODone], 0);
        }
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace ark

using namespace ark;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_prefill_mu;       // guards the per-device set-up below (first calls may come from several threads)
bool g_prefill_attr[64];

}  // namespace

namespace {

ark_status prefill_checks(int B, int S, int T, int Hq, int Hkv, int D, float scale) {
    if (B <= 0 || S <= 0 || T <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || !(scale > 0.f)) return ARK_ERR_INVALID_ARG;
    if (Hq % Hkv != 0) return ARK_ERR_INVALID_ARG;
    if (D != kHeadDim || Hq / Hkv != kGroup) return ARK_ERR_UNSUPPORTED;
    if (T > ARK_MAX_T || B > 65535 || Hkv > 65535) return ARK_ERR_UNSUPPORTED;
    if (static_cast<long long>(B) * S >= (1LL << 31) || static_cast<long long>(B) * T >= (1LL << 31))
        return ARK_ERR_UNSUPPORTED;
    return ARK_OK;
}

// one launch over layers [l0, l0 + n) of the per-layer arrays
ark_status launch_prefill(const void* const* q, const void* const* cache_k, const void* const* cache_v,
                          void* const* o, float* const* lse, int l0, int n, const int32_t* pos0,
                          const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, float scale,
                          const float* table, uint32_t* d_status, cudaStream_t stream) {
    static thread_local pf::Params prm;
    prm = pf::Params{};
    for (int i = 0; i < n; ++i) {
        const int l = l0 + i;
        if (!q[l] || !cache_k[l] || !cache_v[l] || !o[l] || !lse[l]) return ARK_ERR_INVALID_ARG;
        if (!aligned16(q[l]) || !aligned16(cache_k[l]) || !aligned16(cache_v[l]) || !aligned16(o[l]) ||
            (reinterpret_cast<uintptr_t>(lse[l]) & 3u))
            return ARK_ERR_INVALID_ARG;
        if (!q_group_tensor_map(&prm.qmap[i], q[l], static_cast<long long>(B) * S, Hq, 64, pf::kPos) ||
            !kv_tensor_map(&prm.kmap[i], cache_k[l], static_cast<long long>(B) * T, Hkv, 64, pf::kBN) ||
            !kv_tensor_map(&prm.vmap[i], cache_v[l], static_cast<long long>(B) * T, Hkv, 64, pf::kBN) ||
            !q_group_tensor_map(&prm.omap[i], o[l], static_cast<long long>(B) * S, Hq, 64, 1))
            return ARK_ERR_CUDA;
        prm.lse[i] = lse[l];
    }
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv; prm.L = n;
    prm.table = reinterpret_cast<const float4*>(table);
    prm.scale_log2 = scale * kLog2e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(g_prefill_mu);
        if (!g_prefill_attr[dev]) {
            if (cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pf::kSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pf::kSmemBytes) != cudaSuccess)
                return ARK_ERR_CUDA;
            g_prefill_attr[dev] = true;
        }
    }
    const long long ctas = static_cast<long long>(Hkv) * B * ((S + pf::kPos - 1) / pf::kPos) * n;
    if (ctas >= (1LL << 31)) return ARK_ERR_UNSUPPORTED;
    if (table)
        prefill_kernel<true><<<static_cast<unsigned>(ctas), pf::kThreads, pf::kSmemBytes, stream>>>(prm);
    else
        prefill_kernel<false><<<static_cast<unsigned>(ctas), pf::kThreads, pf::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

}  // namespace

extern "C" ark_status ark_attn_prefill(const void* q, const void* cache_k, const void* cache_v,
                                       const int32_t* pos0, const int32_t* n_new, int B, int S, int T, int Hq,
                                       int Hkv, int D, float scale, void* o, float* lse, uint32_t* d_status,
                                       cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !pos0 || !n_new || !o || !lse) return ARK_ERR_INVALID_ARG;
    ark_status st = prefill_checks(B, S, T, Hq, Hkv, D, scale);
    if (st != ARK_OK) return st;
    return launch_prefill(&q, &cache_k, &cache_v, &o, &lse, 0, 1, pos0, n_new, B, S, T, Hq, Hkv, scale, nullptr,
                          d_status, stream);
}

extern "C" ark_status ark_attn_prefill_layers(int L, const void* const* q, const void* const* cache_k,
                                              const void* const* cache_v, const int32_t* pos0,
                                              const int32_t* n_new, int B, int S, int T, int Hq, int Hkv, int D,
                                              float scale, void* const* o, float* const* lse, uint32_t* d_status,
                                              cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !pos0 || !n_new || !o || !lse) return ARK_ERR_INVALID_ARG;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    ark_status st = prefill_checks(B, S, T, Hq, Hkv, D, scale);
    if (st != ARK_OK) return st;
    for (int l0 = 0; l0 < L; l0 += pf::kLayersPerLaunch) {
        const int n = (L - l0 < pf::kLayersPerLaunch) ? L - l0 : pf::kLayersPerLaunch;
        st = launch_prefill(q, cache_k, cache_v, o, lse, l0, n, pos0, n_new, B, S, T, Hq, Hkv, scale, nullptr,
                            d_status, stream);
        if (st != ARK_OK) return st;
    }
    return ARK_OK;
}

extern "C" ark_status ark_attn_prefill_rope_layers(int L, const void* const* q, const void* const* cache_k,
                                                   const void* const* cache_v, const int32_t* pos0,
                                                   const int32_t* n_new, int B, int S, int T, int Hq, int Hkv,
                                                   int D, float scale, const float* d_table, void* const* o,
                                                   float* const* lse, uint32_t* d_status, cudaStream_t stream) {
    if (!q || !cache_k || !cache_v || !pos0 || !n_new || !o || !lse || !d_table) return ARK_ERR_INVALID_ARG;
    if (L <= 0) return ARK_ERR_INVALID_ARG;
    if (L > ARK_MAX_LAYERS) return ARK_ERR_UNSUPPORTED;
    ark_status st = prefill_checks(B, S, T, Hq, Hkv, D, scale);
    if (st != ARK_OK) return st;
    if (!aligned16(d_table)) return ARK_ERR_INVALID_ARG;
    for (int l0 = 0; l0 < L; l0 += pf::kLayersPerLaunch) {
        const int n = (L - l0 < pf::kLayersPerLaunch) ? L - l0 : pf::kLayersPerLaunch;
        st = launch_prefill(q, cache_k, cache_v, o, lse, l0, n, pos0, n_new, B, S, T, Hq, Hkv, scale, d_table,
                            d_status, stream);
        if (st != ARK_OK) return st;
    }
    return ARK_OK;
}

extern "C" ark_status ark_attn_prefill_rope(const void* q, const void* cache_k, const void* cache_v,
                                            const int32_t* pos0, const int32_t* n_new, int B, int S, int T, int Hq,
                                            int Hkv, int D, float scale, const float* d_table, void* o, float* lse,
                                            uint32_t* d_status, cudaStream_t stream) {
    return ark_attn_prefill_rope_layers(1, &q, &cache_k, &cache_v, pos0, n_new, B, S, T, Hq, Hkv, D, scale, d_table,
                                        &o, &lse, d_status, stream);
}
