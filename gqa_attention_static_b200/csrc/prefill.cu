// prefill.cu -- causal GQA prefill of the prompt on the 5th-generation tensor
// cores (tcgen05, accumulators in tensor memory, operands staged by TMA).
//
// The ONNX model card ("ARK-ASR-3B -- INT8 ONNX", sections Shapes and
// Inference) runs the whole audio+text prompt through the decoder in one call
// ("Prefill, then decode"); each call's key/value rows are written into the
// static cache at cache_position.  Here the rows are already appended (by
// ark_attn_append_rope or ark_attn_append_rope_kv) and query row t of request
// b, at absolute position p = pos0[b] + t, attends to the cache rows j <= p of
// its KV head.
//
// Work decomposition (B200):
//   - A tile is 16 query positions x the 8 query heads of one KV group: 128
//     MMA rows, so every K/V block is read once for all 8 heads (GQA packing).
//     A unit is two consecutive tiles A and B (32 positions) of one (layer,
//     request, KV head); they share every K/V block.  Units are ordered by
//     layer chunk, then by decreasing absolute position (longest key range
//     first), then request, KV head and layer, and the kernel is persistent:
//     one CTA per SM walks its units in snake order over that list, so the
//     SMs never drain between layers or tiles.
//   - The units of a CTA form one stream of steps (unit, 64-key block) with no
//     break at unit boundaries: the score MMAs run ahead of the P V MMAs by up
//     to the two S buffers of each tile (possibly into the next unit), and each
//     unit's epilogue runs after the softmax of the next unit's first block, so
//     neither the tensor cores nor the softmax warps wait for a unit to drain.
//   - Warp roles.  Warp 10 computes the unit list entries (a binary search
//     over position levels, from pos0/n_new on the device), publishes them in
//     a 4-entry ring and loads each unit's Q tiles by TMA into one of two Q
//     slots; a slot is reloaded as soon as the last score MMA that reads it has
//     completed.  Warp 0 streams the K and V blocks (64 keys, 16 KB each)
//     through 3-stage rings.  Two warps issue the MMAs, each from one thread:
//     warp 1 the scores S = Q K^T, warp 11 the products O += P V, so that the
//     waits of one chain do not hold up the other (each thread's MMAs complete
//     in issue order, and its commits track only its own).  Warps 2..5 run the
//     softmax and epilogue of tile A, warps 6..9 those of tile B, one thread
//     per row.  With RoPE on load, warps 12..15 rotate the landed Q tiles in
//     shared memory before the first MMA.
//   - Tensor memory (512 columns): for each tile two S buffers of 64 columns
//     (S = Q K^T of a block: 8 MMAs of 128x64x16) and an O accumulator of 128
//     columns (O += P V: 4 MMAs of 128x128x16 with P, bf16, read from tensor
//     memory over its own S columns and V an MN-major shared-memory operand).
//     A unit's last block computes only the 16-key groups that reach into its
//     causal range (fewer score columns, fewer P V steps).
//   - Softmax in the log2 domain with a lazily moved reference max: O is
//     rescaled in tensor memory only when a row's block max exceeds its
//     reference by more than 2^8.  Only blocks that reach past a row's
//     position are masked; V rows past the unit's causal range are zeroed in
//     shared memory before their (zero-weight) use, so garbage past the valid
//     rows cannot turn into NaN.  Rows past n_new[b] are computed on whatever
//     the padded q holds and never written.  The exponent arguments and the
//     row sums are computed on packed fp32 pairs.
//   - Epilogue: O / (sum of the bf16 weights) as bf16, written by each row's
//     thread straight to its 256-byte output row (16-byte stores); lse by plain
//     stores.
//
// Roofline: per request of L prompt rows and per layer, 4096 * L * (L + 1)
// FLOPs (the causal half of QK^T and PV for 16 heads) against 9216 * L bytes
// (q read, o written, K/V rows read once from HBM); at the prompt lengths of
// the coalesced-prefill workload (<= 387) that is HBM-bound.
#include "common.cuh"
#include "tma_host.h"

#include <mutex>

namespace ark {
namespace pf {

constexpr int kRows = 128;               // MMA M: 16 positions x 8 heads
constexpr int kPos = 16;                 // query positions per tile
constexpr int kUnitPos = 32;             // query positions per unit (tiles A and B)
constexpr int kBN = 64;                  // keys per KV block
constexpr int kQHalf = kRows * 128;      // one 64-dim half of a Q tile (16 KB)
constexpr int kQTile = 2 * kQHalf;       // one Q tile (32 KB)
constexpr int kQSlot = 2 * kQTile;       // the two tiles of a unit (64 KB)
constexpr int kQSlots = 2;
constexpr int kKHalf = kBN * 128;        // one 64-dim half of a K or V block (8 KB)
constexpr int kKV = 2 * kKHalf;          // a K or V block (16 KB)
constexpr int kStages = 3;               // K and V ring depth
constexpr int kDescs = 4;                // unit-list entries in flight

// warps
constexpr int kWarpKV = 0;
constexpr int kWarpMMA = 1;              // score MMAs (S = Q K^T); allocates the tensor memory
constexpr int kWarpSoft0 = 2;            // 2..5 tile A, 6..9 tile B
constexpr int kWarpQ = 10;
constexpr int kWarpPV = 11;              // P V MMAs
constexpr int kWarpRot0 = 12;            // 12..15 (RoPE on load only)
constexpr int kThreads = 384;
constexpr int kThreadsRope = 512;
constexpr int kRotThreads = 128;

// shared memory map (the dynamic shared memory base is 1024-aligned)
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQSlots * kQSlot;
constexpr int kOffV = kOffK + kStages * kKV;
constexpr int kOffBar = kOffV + kStages * kKV;
constexpr int kBarDesc = 0;                          // [kDescs] unit-list entry published
constexpr int kBarDescFree = kBarDesc + kDescs;      // [kDescs] entry read by every consumer warp
constexpr int kBarQFull = kBarDescFree + kDescs;     // [kQSlots] Q tiles landed (tx)
constexpr int kBarQRot = kBarQFull + kQSlots;        // [kQSlots] Q tiles rotated (RoPE on load)
constexpr int kBarQEmpty = kBarQRot + kQSlots;       // [kQSlots] every score MMA of the slot's unit done
constexpr int kBarKFull = kBarQEmpty + kQSlots;      // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages;      // [tile][buffer] scores of a block in TMEM
constexpr int kBarPFull = kBarSFull + 4;             // [tile][buffer] P of a block in TMEM (count 128)
constexpr int kBarPvDone = kBarPFull + 4;            // [tile] one phase per PV
constexpr int kBarODone = kBarPvDone + 2;            // [tile] one phase per unit: every MMA of the tile done
constexpr int kBarOEmpty = kBarODone + 2;            // [tile] O read out of TMEM (count 128)
constexpr int kBarSFree = kBarOEmpty + 2;           // [tile][buffer] the PV that read a block's P is done
constexpr int kBarDrain = kBarSFree + 4;             // [issuing warp] MMAs in flight when it gives up
constexpr int kNumBars = kBarDrain + 2;
constexpr int kOffDesc = (kOffBar + kNumBars * 8 + 15) & ~15;
struct UnitDesc {
    int l, b, g, t0;      // layer (of the launch), request, KV head, first position of tile A (call index)
    int nn, p0;           // request's new rows and cache position (clamped)
    int nblk_a, nblk_b;   // 64-key blocks of tile A and of tile B (0: tile B has no live row)
    int end;              // 1: no more units for this CTA
    int pad[3];
};
constexpr int kOffTmemPtr = kOffDesc + kDescs * static_cast<int>(sizeof(UnitDesc));
constexpr int kSmemBytes = kOffTmemPtr + 16;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffBar % 8 == 0 && kOffTmemPtr % 8 == 0, "alignment");

// TMEM columns: S[tile][buffer] at 128 * tile + 64 * buffer, O[tile] at 256 + 128 * tile
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 256;
constexpr uint32_t kTmemCols = 512;

// instruction descriptors (kind::f16): D fp32, A/B bf16, M = 128
constexpr uint32_t kIdescF16 = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 4) << 24);
// QK: N = keys of the block (64, or fewer 16-key groups on a unit's last block), B = K (K-major)
constexpr uint32_t kIdescPV = kIdescF16 | ((128u >> 3) << 17) | (1u << 16);  // N = 128 dims, B = V (MN-major)

constexpr float kLazyRescale = 8.0f;     // log2 units: rescale O only past a factor 2^8

// layers per launch: three tensor maps per layer in the kernel parameters
constexpr int kLayersPerLaunch = 36;
// layers per chunk of the unit order (the K/V rows of a chunk stay in L2 while its units run)
constexpr int kLayerChunk = 12;

struct Params {
    CUtensorMap qmap[kLayersPerLaunch];   // q as (128, 8, Hq/8, B*S), box (64, 8, 1, 16)
    CUtensorMap kmap[kLayersPerLaunch];   // cache_k as (128, Hkv, B*T), box (64, 1, 64)
    CUtensorMap vmap[kLayersPerLaunch];
    __nv_bfloat16* o[kLayersPerLaunch];   // [B, S, Hq, 128]
    float* lse[kLayersPerLaunch];         // [B, Hq, S]
    const int32_t* pos0;
    const int32_t* n_new;
    uint32_t* status;
    const float4* table;                  // rotary table [T][64] {cos, sin} (fp32), for RoPE on load
    int B, S, T, Hq, Hkv, L, Lc;
    int o_align32;                        // every o[l] 32-byte aligned: 32-byte stores
    float scale_log2;
};
static_assert(sizeof(Params) <= 32000, "kernel parameter space");

// Request b's lengths as the kernel uses them (device values, clamped into
// range; `bad` when they had to be), and its units' position levels: unit k
// of request b starts at absolute position pos0 + 32 k, level (pos0 >> 5) + k,
// and the request has ceil(n_new / 32) units.
struct ReqUnits {
    int nn, p0, lev0, nunits;
    bool bad;
};

__device__ __forceinline__ ReqUnits req_units(const Params& p, int b) {
    ReqUnits t;
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
    t.lev0 = p0 >> 5;
    t.nunits = (nn + kUnitPos - 1) / kUnitPos;
    return t;
}

// units of a request at levels >= lam
__device__ __forceinline__ int units_at_or_above(const ReqUnits& t, int lam) {
    const int c = t.lev0 + t.nunits - max(lam, t.lev0);
    return c < 0 ? 0 : c;
}

// (level, request) pairs at levels >= lam, over the whole batch; one warp,
// every lane returns the same count.  `bad` collects clamped requests.
__device__ __forceinline__ int count_units(const Params& p, int lam, int lane, bool& bad) {
    int c = 0;
    for (int b = lane; b < p.B; b += 32) {
        const ReqUnits t = req_units(p, b);
        c += units_at_or_above(t, lam);
        bad |= t.bad;
    }
    return static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(c)));
}

// The j-th (level, request) pair in the order (level descending, request
// ascending), j < count_units(0); one warp, every lane returns the same pair.
// C(lam) = pairs at levels >= lam is non-increasing; the pair's level is the
// largest lam with C(lam) > j.
__device__ __forceinline__ void pick_unit(const Params& p, int j, int lane, int& b_out, int& k_out, ReqUnits& req) {
    const unsigned full = 0xffffffffu;
    bool bad = false;
    int lo = 0, hi = ((p.T - 1) >> 5) + 1;        // C(lo) > j, C(hi) == 0
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (count_units(p, mid, lane, bad) > j) lo = mid;
        else hi = mid;
    }
    int rank = j - count_units(p, lo + 1, lane, bad);   // among the requests with a unit at level lo
    b_out = 0;
    k_out = 0;
    req = ReqUnits{0, 0, 0, 0, false};
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        const ReqUnits t = b < p.B ? req_units(p, b) : ReqUnits{0, 0, 0, 0, false};
        const bool at = b < p.B && t.lev0 <= lo && lo < t.lev0 + t.nunits;
        const unsigned m = __ballot_sync(full, at);
        const int n = __popc(m);
        if (rank < n) {
            const int src = static_cast<int>(__fns(m, 0, rank + 1));
            b_out = base + src;
            req.nn = __shfl_sync(full, t.nn, src);
            req.p0 = __shfl_sync(full, t.p0, src);
            req.lev0 = __shfl_sync(full, t.lev0, src);
            req.nunits = __shfl_sync(full, t.nunits, src);
            k_out = lo - req.lev0;
            return;
        }
        rank -= n;
    }
}

__device__ __forceinline__ int ceil_div(int a, int b) { return (a + b - 1) / b; }

// The k-th unit of CTA c among G CTAs: snake order over the unit list.
__device__ __forceinline__ long long snake_unit(int k, int c, int G) {
    return static_cast<long long>(k) * G + ((k & 1) ? G - 1 - c : c);
}

// Unit-list entry i (one warp, same result in every lane).  The list: layer
// chunks of Lc layers in order; within a chunk, (level, request) pairs by
// decreasing level, then KV heads, then the chunk's layers.
__device__ __forceinline__ UnitDesc unit_desc(const Params& p, long long i, int per_head, long long total, int lane) {
    UnitDesc d{};
    if (i >= total) {
        d.end = 1;
        return d;
    }
    const long long per_chunk = static_cast<long long>(p.Lc) * p.Hkv * per_head;
    const int ch = static_cast<int>(i / per_chunk);
    const long long ii = i - ch * per_chunk;
    const int nlc = min(p.Lc, p.L - ch * p.Lc);
    d.l = ch * p.Lc + static_cast<int>(ii % nlc);
    const long long r = ii / nlc;
    d.g = static_cast<int>(r % p.Hkv);
    const int j = static_cast<int>(r / p.Hkv);
    int b, k;
    ReqUnits t;
    pick_unit(p, j, lane, b, k, t);
    d.b = b;
    d.nn = t.nn;
    d.p0 = t.p0;
    d.t0 = k * kUnitPos;
    const int end_a = t.p0 + min(d.t0 + kPos, t.nn);              // keys visible to tile A's last row
    d.nblk_a = ceil_div(end_a, kBN);
    if (d.t0 + kPos < t.nn) {
        const int end_b = t.p0 + min(d.t0 + kUnitPos, t.nn);
        d.nblk_b = ceil_div(end_b, kBN);
    } else {
        d.nblk_b = 0;
    }
    d.end = 0;
    return d;
}

}  // namespace pf

namespace pf {
// the unit-list fields an MMA warp computes descriptors from, made warp-uniform (broadcast from
// lane 0) so that every lane derives the same descriptor values and one elected lane issues
__device__ __forceinline__ void uniform_desc(UnitDesc& d) {
    d.l = __shfl_sync(0xffffffffu, d.l, 0);
    d.t0 = __shfl_sync(0xffffffffu, d.t0, 0);
    d.nn = __shfl_sync(0xffffffffu, d.nn, 0);
    d.p0 = __shfl_sync(0xffffffffu, d.p0, 0);
    d.nblk_a = __shfl_sync(0xffffffffu, d.nblk_a, 0);
    d.nblk_b = __shfl_sync(0xffffffffu, d.nblk_b, 0);
    d.end = __shfl_sync(0xffffffffu, d.end, 0);
}
}  // namespace pf

template <bool Rope>
__global__ void __launch_bounds__(Rope ? pf::kThreadsRope : pf::kThreads, 1)
    prefill_kernel(const __grid_constant__ pf::Params p) {
    using namespace pf;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const unsigned full = 0xffffffffu;
    if (smem_u32(smem) & 1023u) {                           // the swizzled layouts need 1024-byte alignment
        if (threadIdx.x == 0) report(p.status, ARK_DEV_TIMEOUT);
        return;
    }
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    UnitDesc* descs = reinterpret_cast<UnitDesc*>(smem + kOffDesc);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) {
            uint32_t cnt = 1;
            if ((i >= kBarPFull && i < kBarPFull + 4) || (i >= kBarOEmpty && i < kBarOEmpty + 2)) cnt = kRows;
            if (i >= kBarQRot && i < kBarQRot + kQSlots) cnt = kRotThreads;
            // readers of an entry: the K/V producer, the two MMA warps, 8 softmax warps (+4 rotation warps)
            if (i >= kBarDescFree && i < kBarDescFree + kDescs) cnt = Rope ? 15 : 11;
            mbar_init(&bars[i], cnt);
        }
        fence_mbar_init();
    }
    if (warp == kWarpMMA) tmem_alloc(tmem_ptr, kTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t sbase = smem_u32(smem);

    // the published unit-list entry k (every consumer role waits for it)
    auto wait_desc = [&](int k, UnitDesc& d) -> bool {
        if (!mbar_wait(&bars[kBarDesc + (k & (kDescs - 1))], (k / kDescs) & 1)) return false;
        d = descs[k & (kDescs - 1)];
        return true;
    };
    // a consumer warp has read entry k (one arrival per warp, by lane 0, after the whole warp read it)
    auto free_desc = [&](int k) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[kBarDescFree + (k & (kDescs - 1))]);
    };
    auto fail = [&]() { report(p.status, ARK_DEV_TIMEOUT); };

    if (warp == kWarpQ) {
        // ================================================= unit list, Q loads
        bool ok = true, bad = false;
        const int per_head = count_units(p, 0, lane, bad);
        const bool any_bad = __any_sync(full, bad);
        if (c == 0 && lane == 0 && any_bad) report(p.status, ARK_DEV_BAD_POS);
        const long long total = static_cast<long long>(p.L) * p.Hkv * per_head;
        int q_issued = -1;                    // last unit whose Q was loaded
        for (int k = 0;; ++k) {
            const UnitDesc d = unit_desc(p, snake_unit(k, c, G), per_head, total, lane);
            if (lane == 0) {
                // entry slot k % 4 last held unit k - 4: every consumer warp has read it
                if (k >= kDescs && ok)
                    ok = mbar_wait(&bars[kBarDescFree + (k & (kDescs - 1))], ((k / kDescs) - 1) & 1);
                if (!ok) {
                    // publish the end of the list so that the other roles stop
                    UnitDesc e{};
                    e.end = 1;
                    descs[k & (kDescs - 1)] = e;
                } else {
                    descs[k & (kDescs - 1)] = d;
                }
                mbar_arrive(&bars[kBarDesc + (k & (kDescs - 1))]);
                const int qs = k & 1;
                // the slot last held unit k - 2: its score MMAs have completed
                if (ok && !d.end && k >= 2) ok = mbar_wait(&bars[kBarQEmpty + qs], ((k - 2) >> 1) & 1);
                if (ok && !d.end) {
                    const int ntile = d.nblk_b > 0 ? 2 : 1;
                    mbar_arrive_expect_tx(&bars[kBarQFull + qs], ntile * kQTile);
                    uint8_t* qd = smem + kOffQ + qs * kQSlot;
                    for (int x = 0; x < ntile; ++x) {
                        const int row = d.b * p.S + d.t0 + x * kPos;
                        tma_load_4d(qd + x * kQTile, &p.qmap[d.l], 0, 0, d.g, row, &bars[kBarQFull + qs]);
                        tma_load_4d(qd + x * kQTile + kQHalf, &p.qmap[d.l], 64, 0, d.g, row, &bars[kBarQFull + qs]);
                    }
                    q_issued = k;
                }
            }
            ok = __shfl_sync(full, ok ? 1 : 0, 0) != 0;
            if (d.end || !ok) break;
        }
        if (lane == 0 && !ok) {
            fail();
            // every Q copy issued has landed before the shared memory can go away
            if (q_issued >= 0) (void)mbar_wait(&bars[kBarQFull + (q_issued & 1)], (q_issued >> 1) & 1);
            if (q_issued >= 1)
                (void)mbar_wait(&bars[kBarQFull + ((q_issued - 1) & 1)], ((q_issued - 1) >> 1) & 1);
        }
        __syncwarp();
    } else if (warp == kWarpKV) {
        // ================================================= K/V producer
        if (lane == 0) {
            bool ok = true;
            int gk = 0;                                        // blocks issued so far
            for (int k = 0; ok; ++k) {
                UnitDesc d;
                if (!(ok = wait_desc(k, d))) break;
                mbar_arrive(&bars[kBarDescFree + (k & (kDescs - 1))]);
                if (d.end) break;
                const int nb = max(d.nblk_a, d.nblk_b);
                const int row0 = d.b * p.T;
                for (int j = 0; j < nb; ++j, ++gk) {
                    const int st = gk % kStages;
                    const uint32_t par = ((gk / kStages) - 1) & 1;
                    if (gk >= kStages && !(ok = mbar_wait(&bars[kBarKEmpty + st], par))) break;
                    mbar_arrive_expect_tx(&bars[kBarKFull + st], kKV);
                    uint8_t* kd = smem + kOffK + st * kKV;
                    tma_load_3d(kd, &p.kmap[d.l], 0, d.g, row0 + j * kBN, &bars[kBarKFull + st]);
                    tma_load_3d(kd + kKHalf, &p.kmap[d.l], 64, d.g, row0 + j * kBN, &bars[kBarKFull + st]);
                    if (gk >= kStages && !(ok = mbar_wait(&bars[kBarVEmpty + st], par))) {
                        ++gk;                                  // the K copy of this block is in flight
                        break;
                    }
                    mbar_arrive_expect_tx(&bars[kBarVFull + st], kKV);
                    uint8_t* vd = smem + kOffV + st * kKV;
                    tma_load_3d(vd, &p.vmap[d.l], 0, d.g, row0 + j * kBN, &bars[kBarVFull + st]);
                    tma_load_3d(vd + kKHalf, &p.vmap[d.l], 64, d.g, row0 + j * kBN, &bars[kBarVFull + st]);
                }
            }
            if (!ok) {
                fail();
                // every copy issued has landed before the shared memory can go away
                for (int g2 = max(0, gk - kStages); g2 < gk; ++g2) {
                    (void)mbar_wait(&bars[kBarKFull + g2 % kStages], (g2 / kStages) & 1);
                    (void)mbar_wait(&bars[kBarVFull + g2 % kStages], (g2 / kStages) & 1);
                }
            }
        }
    } else if (warp == kWarpMMA) {
        // ================================================= score MMAs (S = Q K^T)
        // Runs ahead of the softmax by up to the two S buffers of each tile: a buffer is reused once
        // the PV that read its P has completed.  Waits are AND-ed over the warp so that the
        // __syncwarp()s below are reached by all lanes.
        bool ok = true;
        int sq[2] = {0, 0};       // QK blocks issued per tile (S buffer = sq & 1)
        int g = 0;                // K/V blocks consumed
        // descriptors of the shared-memory operands at the region bases; offsets are added in 16-byte units
        const uint64_t dq0 = umma_desc_sw128(sbase + kOffQ, 16, 1024);
        const uint64_t dk0 = umma_desc_sw128(sbase + kOffK, 16, 1024);
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(full, wait_desc(k, d)))) break;
            free_desc(k);
            uniform_desc(d);
            if (d.end) break;
            if (!(ok = __all_sync(full, mbar_wait(&bars[(Rope ? kBarQRot : kBarQFull) + (k & 1)], (k >> 1) & 1))))
                break;
            const int nbx[2] = {d.nblk_a, d.nblk_b};
            const int nb = max(d.nblk_a, d.nblk_b);
            const int kv_end = d.p0 + min(d.t0 + (d.nblk_b > 0 ? kUnitPos : kPos), d.nn);
            const uint64_t qslot = dq0 + static_cast<uint64_t>(((k & 1) * kQSlot) >> 4);
            for (int j = 0; j < nb && ok; ++j, ++g) {
                const int st = g % kStages;
                if (!(ok = __all_sync(full, mbar_wait(&bars[kBarKFull + st], (g / kStages) & 1)))) break;
                for (int x = 0; x < 2 && ok; ++x)
                    if (j < nbx[x] && sq[x] >= 2)
                        ok = __all_sync(full, mbar_wait(&bars[kBarSFree + x * 2 + (sq[x] & 1)],
                                                        ((sq[x] >> 1) - 1) & 1));
                if (!ok) break;
                // scores past the unit's causal range are masked by the softmax: the last block computes
                // only the 16-key groups that reach into the range (the columns past them are never used
                // unmasked)
                const int n16 = min(kBN, (kv_end - j * kBN + 15) & ~15);
                const uint32_t idesc = kIdescF16 | (static_cast<uint32_t>(n16 >> 3) << 17);
                // the whole warp computes the (uniform) descriptors; one elected lane issues each instruction
                tc_fence_after();
                const uint64_t kb = dk0 + static_cast<uint64_t>((st * kKV) >> 4);
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    if (j >= nbx[x]) continue;
                    const uint32_t dcol = tmem + kColS + x * 128 + (sq[x] & 1) * kBN;
                    const uint64_t qa = qslot + static_cast<uint64_t>((x * kQTile) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kQHalf + (kk & 3) * 32) >> 4);
                        const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * kKHalf + (kk & 3) * 32) >> 4);
                        if (elect_one()) umma_f16(dcol, qa + off, kb + koff, idesc, kk > 0 ? 1u : 0u);
                    }
                    if (elect_one()) umma_commit(&bars[kBarSFull + x * 2 + (sq[x] & 1)]);
                }
                if (elect_one()) umma_commit(&bars[kBarKEmpty + st]);
                // the unit's last score MMAs: its Q slot may take another unit once they complete
                if (j == nb - 1 && elect_one()) umma_commit(&bars[kBarQEmpty + (k & 1)]);
                __syncwarp();
                for (int x = 0; x < 2; ++x)
                    if (j < nbx[x]) ++sq[x];
            }
        }
        if (!ok) {
            if (lane == 0) {
                fail();
                umma_commit(&bars[kBarDrain]);
                (void)mbar_wait(&bars[kBarDrain], 0);            // MMAs issued so far have completed
            }
            __syncwarp();
        }
    } else if (warp == kWarpPV) {
        // ================================================= P V MMAs (O += P V)
        bool ok = true;
        int pv[2] = {0, 0};       // PV blocks issued per tile (P buffer = pv & 1)
        int uo[2] = {0, 0};       // units whose last PV was issued, per tile (O phases)
        int g = 0;                // K/V blocks consumed
        const uint64_t dv0 = umma_desc_sw128(sbase + kOffV, kKHalf, 1024);
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(full, wait_desc(k, d)))) break;
            free_desc(k);
            uniform_desc(d);
            if (d.end) break;
            const int nbx[2] = {d.nblk_a, d.nblk_b};
            const int nb = max(d.nblk_a, d.nblk_b);
            const int kv_end = d.p0 + min(d.t0 + (d.nblk_b > 0 ? kUnitPos : kPos), d.nn);
            for (int j = 0; j < nb && ok; ++j, ++g) {
                const int st = g % kStages;
                if (!(ok = __all_sync(full, mbar_wait(&bars[kBarVFull + st], (g / kStages) & 1)))) break;
                const int live = min(kBN, kv_end - j * kBN);      // rows of the block inside the causal range
                const int ksteps = min(kBN, (live + 15) & ~15) >> 4;   // 16-row groups that reach into it
                if (live < ksteps * 16) {
                    // the rows of the last group past the range may hold anything (NaN included): P is 0
                    // there, 0 * NaN is not
                    uint8_t* vt = smem + kOffV + st * kKV;
                    for (int i = lane; i < (ksteps * 16 - live) * 16; i += 32) {
                        const int r = live + (i >> 4), part = i & 15;
                        *reinterpret_cast<uint4*>(vt + (part >> 3) * kKHalf + r * 128 + (part & 7) * 16) =
                            make_uint4(0, 0, 0, 0);
                    }
                    fence_proxy_async_smem();
                }
                __syncwarp();
                for (int x = 0; x < 2 && ok; ++x) {
                    if (j >= nbx[x]) continue;
                    // the first PV of a unit overwrites O_x: the previous unit's epilogue must have read it
                    if (j == 0 && uo[x] > 0 &&
                        !(ok = __all_sync(full, mbar_wait(&bars[kBarOEmpty + x], (uo[x] - 1) & 1))))
                        break;
                    if (!(ok = __all_sync(full, mbar_wait(&bars[kBarPFull + x * 2 + (pv[x] & 1)], (pv[x] >> 1) & 1))))
                        break;
                    const bool last = j == nbx[x] - 1;
                    tc_fence_after();
                    const uint32_t pa = tmem + kColS + x * 128 + (pv[x] & 1) * kBN;   // P: 32 columns
                    const uint64_t vb = dv0 + static_cast<uint64_t>((st * kKV) >> 4);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        if (kk < ksteps && elect_one())
                            umma_f16_ts(tmem + kColO + x * 128, pa + kk * 8, vb + static_cast<uint64_t>(kk * 128),
                                        kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);   // 16 V rows = 2048 bytes
                    if (elect_one()) {
                        umma_commit(&bars[kBarPvDone + x]);
                        umma_commit(&bars[kBarSFree + x * 2 + (pv[x] & 1)]);
                        if (last) umma_commit(&bars[kBarODone + x]);
                    }
                    __syncwarp();
                    ++pv[x];
                    if (last) ++uo[x];
                }
                if (!ok) break;
                if (elect_one()) umma_commit(&bars[kBarVEmpty + st]);
                __syncwarp();
            }
        }
        if (!ok) {
            if (lane == 0) {
                fail();
                umma_commit(&bars[kBarDrain + 1]);
                (void)mbar_wait(&bars[kBarDrain + 1], 0);        // MMAs issued so far have completed
            }
            __syncwarp();
        }
    } else if (warp >= kWarpSoft0 && warp < kWarpQ) {
        // ================================================= softmax + epilogue of tile x
        const int x = (warp - kWarpSoft0) >> 2;         // 0: tile A (warps 2..5), 1: tile B (warps 6..9)
        const int quad = warp & 3;                      // TMEM lanes 32*quad .. +31
        const int r = quad * 32 + lane;                 // this thread's row of the tile
        const int hh = r & 7;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t col_s = kColS + x * 128;
        const uint32_t col_o = kColO + x * 128;
        const float sl2 = p.scale_log2;
        const uint64_t sl2x2 = f2_make(sl2, sl2);
        bool ok = true;
        int sq = 0;               // blocks processed (S/P buffer = sq & 1; also the PV count)
        int uo = 0;               // units finished (O phases)
        // the unit whose output still sits in O_x: its epilogue runs after the next unit's first block
        bool pend = false;
        int e_l = 0, e_b = 0, e_g = 0, e_tr = 0, e_nn = 0;
        float e_m = 0.f, e_sum = 0.f, e_rsum = 1.f;
        auto epilogue = [&]() -> bool {
            if (!__all_sync(full, mbar_wait(&bars[kBarODone + x], uo & 1))) return false;
            ++uo;
            tc_fence_after();
            const float inv = 1.f / e_rsum;
            // O row as bf16 pairs: read all of it before releasing O_x to the next unit's first PV
            uint32_t w[64];
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                uint32_t o[64];
                tmem_ld32(lane_base + col_o + 64 * c2, *reinterpret_cast<uint32_t(*)[32]>(o));
                tmem_ld32(lane_base + col_o + 64 * c2 + 32, *reinterpret_cast<uint32_t(*)[32]>(o + 32));
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    w[32 * c2 + i] = cvt_bf16x2(__uint_as_float(o[2 * i]) * inv, __uint_as_float(o[2 * i + 1]) * inv);
            }
            tc_fence_before();
            mbar_arrive(&bars[kBarOEmpty + x]);                // the next unit may overwrite O_x
            if (e_tr < e_nn) {
                const int h = e_g * kGroup + hh;
                uint8_t* dst = reinterpret_cast<uint8_t*>(p.o[e_l]) +
                               ((static_cast<size_t>(e_b) * p.S + e_tr) * p.Hq + h) * (kHeadDim * 2);
                if (p.o_align32) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) st_global_v8(dst + 32 * q, &w[8 * q]);
                } else {
#pragma unroll
                    for (int q = 0; q < 16; ++q) st_global_v4(dst + 16 * q, w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                }
                p.lse[e_l][(static_cast<size_t>(e_b) * p.Hq + h) * p.S + e_tr] = (e_m + __log2f(e_sum)) * kLn2;
            }
            return true;
        };
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(full, wait_desc(k, d)))) break;
            free_desc(k);
            if (d.end) break;
            const int nbl = x ? d.nblk_b : d.nblk_a;
            if (nbl == 0) continue;                      // tile B of this unit has no live row
            const int tr = d.t0 + x * kPos + (r >> 3);   // this row's position (call index)
            const int prow = d.p0 + tr;                  // and its absolute position
            float m_ref = -INFINITY;
            uint64_t esum = f2_make(0.f, 0.f), rsum = f2_make(0.f, 0.f);
            // every tcgen05.ld/st is .sync.aligned and sits on warp-uniform control flow
            for (int j = 0; j < nbl; ++j, ++sq) {
                const int buf = sq & 1;
                if (!(ok = __all_sync(full, mbar_wait(&bars[kBarSFull + x * 2 + buf], (sq >> 1) & 1)))) break;
                tc_fence_after();
                const uint32_t scol = lane_base + col_s + buf * kBN;
                uint32_t v[64];
                tmem_ld32(scol, *reinterpret_cast<uint32_t(*)[32]>(v));
                tmem_ld32(scol + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
                tmem_wait_ld();
                const int nvalid = prow - j * kBN + 1;          // keys of this block the row sees
                if (nvalid < kBN) {
#pragma unroll
                    for (int i = 0; i < 64; ++i)
                        if (i >= nvalid) v[i] = 0xff800000u;    // -inf
                }
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                for (int i = 0; i < 64; i += 8) {
                    mx[0] = fmax3(mx[0], __uint_as_float(v[i + 0]), __uint_as_float(v[i + 1]));
                    mx[1] = fmax3(mx[1], __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
                    mx[2] = fmax3(mx[2], __uint_as_float(v[i + 4]), __uint_as_float(v[i + 5]));
                    mx[3] = fmax3(mx[3], __uint_as_float(v[i + 6]), __uint_as_float(v[i + 7]));
                }
                const float bm = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * sl2;
                float alpha = 1.f;
                bool rescale = false;
                if (m_ref == -INFINITY) {
                    m_ref = bm;                 // first block of this row: O is still empty
                } else if (bm > m_ref + kLazyRescale) {
                    alpha = fast_exp2(m_ref - bm);
                    m_ref = bm;
                    rescale = true;
                }
                const float mu = (m_ref == -INFINITY) ? 0.f : m_ref;
                const bool any_rescale = __any_sync(full, rescale);
                if (any_rescale) {
                    const uint64_t a2 = f2_make(alpha, alpha), z2 = f2_make(0.f, 0.f);
                    esum = f2_fma(esum, a2, z2);
                    rsum = f2_fma(rsum, a2, z2);
                }
                // P = exp2(s * scale_log2 - mu) as bf16 pairs: keys 2c, 2c+1 in column c of the block's S
                // buffer (columns 0..31; the scores there are already in registers)
                const uint64_t nmu = f2_make(-mu, -mu);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float a0, a1;
                        f2_split(f2_fma(f2_make(__uint_as_float(v[32 * h2 + 2 * i]),
                                                __uint_as_float(v[32 * h2 + 2 * i + 1])), sl2x2, nmu), a0, a1);
                        const float s0 = fast_exp2(a0), s1 = fast_exp2(a1);
                        const uint32_t w = cvt_bf16x2(s0, s1);
                        esum = f2_add(esum, f2_make(s0, s1));
                        rsum = f2_add(rsum, f2_make(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u)));
                        pk[i] = w;
                    }
                    tmem_st16(scol + 16 * h2, pk);
                }
                if (any_rescale) {
                    // O must hold the PV of every earlier block of the unit (the one before this block
                    // may still run: QK of this block was issued before it) and is rescaled before
                    // this block's P is released to the MMA warp
                    if (!(ok = __all_sync(full, mbar_wait(&bars[kBarPvDone + x], (sq - 1) & 1)))) break;
                    tc_fence_after();
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
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
                mbar_arrive(&bars[kBarPFull + x * 2 + buf]);
                // the previous unit's output, now that this unit's first P is on its way
                if (j == 0 && pend) {
                    if (!(ok = epilogue())) break;
                    pend = false;
                }
            }
            if (!ok) break;
            float e0, e1, r0, r1;
            f2_split(esum, e0, e1);
            f2_split(rsum, r0, r1);
            pend = true;
            e_l = d.l;
            e_b = d.b;
            e_g = d.g;
            e_tr = tr;
            e_nn = d.nn;
            e_m = m_ref;
            e_sum = e0 + e1;
            e_rsum = r0 + r1;
        }
        if (ok && pend) ok = epilogue();
        if (!ok && lane == 0) fail();
    } else if (Rope) {
        // ================================================= RoPE on the landed Q tiles
        // item = (tile, position, 16-byte chunk c, head): the chunk holds dims 8c..8c+7 of the first
        // half and their rotary partners 64 + 8c.. of the second, at the same swizzled offset
        const int tid = threadIdx.x - kWarpRot0 * 32;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(0xffffffffu, wait_desc(k, d)))) break;
            free_desc(k);
            if (d.end) break;
            const int qs = k & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarQFull + qs], (k >> 1) & 1)))) break;
            const int ntile = d.nblk_b > 0 ? 2 : 1;
            for (int it = tid; it < ntile * kPos * 8; it += kRotThreads) {
                const int xt = it / (kPos * 8), rem = it - xt * (kPos * 8);
                const int pp = rem >> 3, cch = rem & 7;
                const int t = d.t0 + xt * kPos + pp;
                if (t >= d.nn) continue;                                   // padded rows are never stored
                const int pos = d.p0 + t;
                double cs[8], sn[8];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float4 tv = __ldg(p.table + static_cast<size_t>(pos) * 32 + 4 * cch + j);  // pairs 2j, 2j+1
                    cs[2 * j] = tv.x; sn[2 * j] = tv.y; cs[2 * j + 1] = tv.z; sn[2 * j + 1] = tv.w;
                }
                uint8_t* base = smem + kOffQ + qs * kQSlot + xt * kQTile;
#pragma unroll 2
                for (int hd = 0; hd < 8; ++hd) {
                    const int rr = pp * 8 + hd;
                    const uint32_t off = rr * 128 + ((cch ^ (rr & 7)) << 4);
                    uint4* plo = reinterpret_cast<uint4*>(base + off);
                    uint4* phi = reinterpret_cast<uint4*>(base + kQHalf + off);
                    const uint4 xlo = *plo, xhi = *phi;
                    const uint32_t wl[4] = {xlo.x, xlo.y, xlo.z, xlo.w}, wh[4] = {xhi.x, xhi.y, xhi.z, xhi.w};
                    uint32_t ol[4], oh[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const double a0 = bf16_bits_to_f64(static_cast<uint16_t>(wl[j] & 0xffff));
                        const double a1 = bf16_bits_to_f64(static_cast<uint16_t>(wl[j] >> 16));
                        const double h0 = bf16_bits_to_f64(static_cast<uint16_t>(wh[j] & 0xffff));
                        const double h1 = bf16_bits_to_f64(static_cast<uint16_t>(wh[j] >> 16));
                        // both products are exact in double, so contraction cannot change the result
                        ol[j] = static_cast<uint32_t>(f64_to_bf16_rn(a0 * cs[2 * j] - h0 * sn[2 * j])) |
                                (static_cast<uint32_t>(f64_to_bf16_rn(a1 * cs[2 * j + 1] - h1 * sn[2 * j + 1])) << 16);
                        oh[j] = static_cast<uint32_t>(f64_to_bf16_rn(h0 * cs[2 * j] + a0 * sn[2 * j])) |
                                (static_cast<uint32_t>(f64_to_bf16_rn(h1 * cs[2 * j + 1] + a1 * sn[2 * j + 1])) << 16);
                    }
                    *plo = make_uint4(ol[0], ol[1], ol[2], ol[3]);
                    *phi = make_uint4(oh[0], oh[1], oh[2], oh[3]);
                }
            }
            fence_proxy_async_smem();                          // the MMA reads the tile through the async proxy
            mbar_arrive(&bars[kBarQRot + qs]);
        }
        if (!ok && (threadIdx.x & 31) == 0) fail();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kWarpMMA) {
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
int g_prefill_sms[64];

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
            !kv_tensor_map(&prm.vmap[i], cache_v[l], static_cast<long long>(B) * T, Hkv, 64, pf::kBN))
            return ARK_ERR_CUDA;
        prm.o[i] = static_cast<__nv_bfloat16*>(o[l]);
        prm.lse[i] = lse[l];
    }
    prm.o_align32 = 1;
    for (int i = 0; i < n; ++i)
        if (reinterpret_cast<uintptr_t>(o[l0 + i]) & 31u) prm.o_align32 = 0;
    prm.pos0 = pos0;
    prm.n_new = n_new;
    prm.status = d_status;
    prm.B = B; prm.S = S; prm.T = T; prm.Hq = Hq; prm.Hkv = Hkv; prm.L = n;
    prm.Lc = n < pf::kLayerChunk ? n : pf::kLayerChunk;
    prm.table = reinterpret_cast<const float4*>(table);
    prm.scale_log2 = scale * kLog2e;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    int sms = 0;
    {
        std::lock_guard<std::mutex> lk(g_prefill_mu);
        if (!g_prefill_attr[dev]) {
            if (cudaFuncSetAttribute(prefill_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pf::kSmemBytes) != cudaSuccess ||
                cudaFuncSetAttribute(prefill_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     pf::kSmemBytes) != cudaSuccess)
                return ARK_ERR_CUDA;
            int nsm = 0;
            if (cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || nsm <= 0)
                return ARK_ERR_CUDA;
            g_prefill_sms[dev] = nsm;
            g_prefill_attr[dev] = true;
        }
        sms = g_prefill_sms[dev];
    }
    // persistent: one CTA per SM, at most one per possible unit
    const long long units_max = static_cast<long long>(n) * Hkv * B * ((S + pf::kUnitPos - 1) / pf::kUnitPos);
    const int grid = static_cast<int>(units_max < sms ? units_max : sms);
    if (table)
        prefill_kernel<true><<<grid, pf::kThreadsRope, pf::kSmemBytes, stream>>>(prm);
    else
        prefill_kernel<false><<<grid, pf::kThreads, pf::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

// L layers in as few launches as the parameter space allows, of near-equal size
ark_status launch_prefill_layers(int L, const void* const* q, const void* const* cache_k, const void* const* cache_v,
                                 void* const* o, float* const* lse, const int32_t* pos0, const int32_t* n_new, int B,
                                 int S, int T, int Hq, int Hkv, float scale, const float* table, uint32_t* d_status,
                                 cudaStream_t stream) {
    const int launches = (L + pf::kLayersPerLaunch - 1) / pf::kLayersPerLaunch;
    for (int i = 0, l0 = 0; i < launches; ++i) {
        const int n = (L - l0) / (launches - i);
        const ark_status st = launch_prefill(q, cache_k, cache_v, o, lse, l0, n, pos0, n_new, B, S, T, Hq, Hkv,
                                             scale, table, d_status, stream);
        if (st != ARK_OK) return st;
        l0 += n;
    }
    return ARK_OK;
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
    return launch_prefill_layers(L, q, cache_k, cache_v, o, lse, pos0, n_new, B, S, T, Hq, Hkv, scale, nullptr,
                                 d_status, stream);
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
    return launch_prefill_layers(L, q, cache_k, cache_v, o, lse, pos0, n_new, B, S, T, Hq, Hkv, scale, d_table,
                                 d_status, stream);
}

extern "C" ark_status ark_attn_prefill_rope(const void* q, const void* cache_k, const void* cache_v,
                                            const int32_t* pos0, const int32_t* n_new, int B, int S, int T, int Hq,
                                            int Hkv, int D, float scale, const float* d_table, void* o, float* lse,
                                            uint32_t* d_status, cudaStream_t stream) {
    return ark_attn_prefill_rope_layers(1, &q, &cache_k, &cache_v, pos0, n_new, B, S, T, Hq, Hkv, D, scale, d_table,
                                        &o, &lse, d_status, stream);
}
