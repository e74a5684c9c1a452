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
//   - Warp roles.  Warp 10 computes the unit list entries (a binary search
//     over position levels, from pos0/n_new on the device), publishes them in
//     a 4-entry ring, loads each unit's Q tiles by TMA into one of two Q slots
//     (so the next unit's Q streams in while this one computes), and issues
//     the TMA stores of each finished unit's output.  Warp 0 streams the K and
//     V blocks (64 keys, 16 KB each) through 3-stage rings.  Warp 1 issues the
//     MMAs from one thread.  Warps 2..5 run the softmax and epilogue of tile A,
//     warps 6..9 those of tile B, one thread per row.  With RoPE on load, warps
//     11..14 rotate the landed Q tiles in shared memory before the first MMA.
//   - Tensor memory (512 columns): for each tile two S buffers of 64 columns
//     (S = Q K^T of a block: 8 MMAs of 128x64x16) and an O accumulator of 128
//     columns (O += P V: 4 MMAs of 128x128x16 with P, bf16, read from tensor
//     memory over its own S columns and V an MN-major shared-memory operand).
//     The MMA warp runs QK of block j+1 ahead of PV of block j, so the softmax
//     of one block overlaps the scores of the next and the other tile's work.
//   - Softmax in the log2 domain with a lazily moved reference max: O is
//     rescaled in tensor memory only when a row's block max exceeds its
//     reference by more than 2^8.  Only blocks that reach past a row's
//     position are masked; V rows past the unit's causal range are zeroed in
//     shared memory before their (zero-weight) use, so garbage past the valid
//     rows cannot turn into NaN.  Rows past n_new[b] are computed on whatever
//     the padded q holds and never written.
//   - Epilogue: O / (sum of the bf16 weights) as bf16 into the unit's finished
//     Q tile in shared memory (the layout of the Q load), then warp 10 stores
//     it by TMA: one box per 64-dim half for a tile whose 16 positions are all
//     live, one box per live position otherwise.  lse by plain stores.
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
constexpr int kWarpMMA = 1;
constexpr int kWarpSoft0 = 2;            // 2..5 tile A, 6..9 tile B
constexpr int kWarpQ = 10;
constexpr int kWarpRot0 = 11;            // 11..14 (RoPE on load only)
constexpr int kThreads = 352;
constexpr int kThreadsRope = 480;
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
constexpr int kBarKFull = kBarQRot + kQSlots;        // [kStages]
constexpr int kBarKEmpty = kBarKFull + kStages;
constexpr int kBarVFull = kBarKEmpty + kStages;
constexpr int kBarVEmpty = kBarVFull + kStages;
constexpr int kBarSFull = kBarVEmpty + kStages;      // [tile][buffer] scores of a block in TMEM
constexpr int kBarPFull = kBarSFull + 4;             // [tile][buffer] P of a block in TMEM (count 128)
constexpr int kBarPvDone = kBarPFull + 4;            // [tile] one phase per PV
constexpr int kBarODone = kBarPvDone + 2;            // [tile] one phase per unit: every MMA of the tile done
constexpr int kBarOEmpty = kBarODone + 2;            // [tile] O read out of TMEM (count 128)
// [tile][Q slot] O staged in shared memory (count 128).  One per slot: the
// softmax warps may finish two consecutive units before warp 10 flushes the
// first, but never two units of the same slot (the slot's next unit needs Q
// tiles that are loaded only after the flush), so each barrier stays within
// one phase of its waiter.
constexpr int kBarStaged = kBarOEmpty + 2;
constexpr int kBarDrain = kBarStaged + 4;            // MMAs in flight when the MMA warp gives up
constexpr int kNumBars = kBarDrain + 1;
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
constexpr uint32_t kIdescQK = kIdescF16 | ((64u >> 3) << 17);                // N = 64 keys, B = K (K-major)
constexpr uint32_t kIdescPV = kIdescF16 | ((128u >> 3) << 17) | (1u << 16);  // N = 128 dims, B = V (MN-major)

constexpr float kLazyRescale = 8.0f;     // log2 units: rescale O only past a factor 2^8

// layers per launch: five tensor maps per layer in the kernel parameters
constexpr int kLayersPerLaunch = 36;
// layers per chunk of the unit order (the K/V rows of a chunk stay in L2 while its units run)
constexpr int kLayerChunk = 12;

struct Params {
    CUtensorMap qmap[kLayersPerLaunch];   // q as (128, 8, Hq/8, B*S), box (64, 8, 1, 16)
    CUtensorMap kmap[kLayersPerLaunch];   // cache_k as (128, Hkv, B*T), box (64, 1, 64)
    CUtensorMap vmap[kLayersPerLaunch];
    CUtensorMap omap[kLayersPerLaunch];   // o as q, box (64, 8, 1, 16): a tile's 64-dim half
    CUtensorMap omap1[kLayersPerLaunch];  // o as q, box (64, 8, 1, 1): one position
    float* lse[kLayersPerLaunch];         // [B, Hq, S]
    const int32_t* pos0;
    const int32_t* n_new;
    uint32_t* status;
    const float4* table;                  // rotary table [T][64] {cos, sin} (fp32), for RoPE on load
    int B, S, T, Hq, Hkv, L, Lc;
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

template <bool Rope>
__global__ void __launch_bounds__(Rope ? pf::kThreadsRope : pf::kThreads, 1)
    prefill_kernel(const __grid_constant__ pf::Params p) {
    using namespace pf;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
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
            if ((i >= kBarPFull && i < kBarPFull + 4) || (i >= kBarOEmpty && i < kBarOEmpty + 2) ||
                (i >= kBarStaged && i < kBarStaged + 4))
                cnt = kRows;
            if (i >= kBarQRot && i < kBarQRot + kQSlots) cnt = kRotThreads;
            // readers of an entry: the K/V producer, the MMA warp, 8 softmax warps (+4 rotation warps)
            if (i >= kBarDescFree && i < kBarDescFree + kDescs) cnt = Rope ? 14 : 10;
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
        // ================================================= unit list, Q loads, O stores
        bool ok = true, bad = false;
        const int per_head = count_units(p, 0, lane, bad);
        const bool any_bad = __any_sync(0xffffffffu, bad);
        if (c == 0 && lane == 0 && any_bad) report(p.status, ARK_DEV_BAD_POS);
        const long long total = static_cast<long long>(p.L) * p.Hkv * per_head;
        int staged[4] = {0, 0, 0, 0};         // [tile][slot]: stagings of tile X in slot s consumed
        UnitDesc prev[2];                     // entries of units k-1, k-2 (ring by k & 1)
        // store the finished output of unit u (its Q slot u & 1), then free that slot
        auto flush = [&](int u, const UnitDesc& d) {
            const int ntile = d.nblk_b > 0 ? 2 : 1;
            for (int x = 0; x < ntile && ok; ++x) {
                const int sb = x * 2 + (u & 1);
                if (!(ok = mbar_wait(&bars[kBarStaged + sb], staged[sb] & 1))) break;
                ++staged[sb];
                const int t0 = d.t0 + x * kPos;
                const int live = min(kPos, d.nn - t0);
                const uint8_t* st = smem + kOffQ + (u & 1) * kQSlot + x * kQTile;
                const int row = d.b * p.S + t0;
                if (live == kPos) {
                    tma_store_4d(&p.omap[d.l], st, 0, 0, d.g, row);
                    tma_store_4d(&p.omap[d.l], st + kQHalf, 64, 0, d.g, row);
                } else {
                    for (int pp = 0; pp < live; ++pp) {
                        tma_store_4d(&p.omap1[d.l], st + pp * 1024, 0, 0, d.g, row + pp);
                        tma_store_4d(&p.omap1[d.l], st + kQHalf + pp * 1024, 64, 0, d.g, row + pp);
                    }
                }
            }
            bulk_commit();
            bulk_wait_read();                 // the slot may take the next Q tiles
        };
        int k = 0;
        int q_issued = -1;                    // last unit whose Q was loaded
        for (;; ++k) {
            const UnitDesc d = unit_desc(p, snake_unit(k, c, G), per_head, total, lane);
            if (lane == 0) {
                if (k >= 2 && ok) flush(k - 2, prev[k & 1]);
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
                if (ok && !d.end) {
                    const int qs = k & 1;
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
                prev[k & 1] = d;
            }
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (d.end || !ok) break;
        }
        if (lane == 0) {
            if (ok && k >= 1 && !prev[(k - 1) & 1].end) flush(k - 1, prev[(k - 1) & 1]);
            if (!ok) {
                fail();
                // every Q copy issued has landed before the shared memory can go away
                if (q_issued >= 0) (void)mbar_wait(&bars[kBarQFull + (q_issued & 1)], (q_issued >> 1) & 1);
                if (q_issued >= 1)
                    (void)mbar_wait(&bars[kBarQFull + ((q_issued - 1) & 1)], ((q_issued - 1) >> 1) & 1);
            }
            bulk_wait_read();
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
        // ================================================= MMA issuer
        // waits are AND-ed over the warp so that the __syncwarp()s below are reached by all lanes
        bool ok = true;
        int sq[2] = {0, 0};       // QK blocks issued per tile (S buffer = sq & 1)
        int pv[2] = {0, 0};       // PV blocks issued per tile (P buffer = pv & 1)
        int uo[2] = {0, 0};       // units finished per tile (O phases)
        int gk = 0;               // K/V blocks consumed
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(0xffffffffu, wait_desc(k, d)))) break;
            free_desc(k);
            if (d.end) break;
            const int qs = k & 1;
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[(Rope ? kBarQRot : kBarQFull) + qs], (k >> 1) & 1))))
                break;
            const int nbx[2] = {d.nblk_a, d.nblk_b};
            const int nb = max(d.nblk_a, d.nblk_b);
            const int kv_end = d.p0 + min(d.t0 + (d.nblk_b > 0 ? kUnitPos : kPos), d.nn);
            const int g0 = gk;
            auto issue_qk = [&](int j) -> bool {
                const int st = (g0 + j) % kStages;
                if (!__all_sync(0xffffffffu, mbar_wait(&bars[kBarKFull + st], ((g0 + j) / kStages) & 1)))
                    return false;
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t kb = sbase + kOffK + st * kKV;
                    for (int x = 0; x < 2; ++x) {
                        if (j >= nbx[x]) continue;
                        const uint32_t dcol = tmem + kColS + x * 128 + (sq[x] & 1) * kBN;
                        const uint32_t qa = sbase + kOffQ + qs * kQSlot + x * kQTile;
#pragma unroll
                        for (int kk = 0; kk < 8; ++kk) {
                            const uint32_t sub = (kk & 3) * 32;
                            umma_f16(dcol, umma_desc_sw128(qa + (kk >> 2) * kQHalf + sub, 16, 1024),
                                     umma_desc_sw128(kb + (kk >> 2) * kKHalf + sub, 16, 1024), kIdescQK,
                                     kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&bars[kBarSFull + x * 2 + (sq[x] & 1)]);
                    }
                    umma_commit(&bars[kBarKEmpty + st]);
                }
                __syncwarp();
                for (int x = 0; x < 2; ++x)
                    if (j < nbx[x]) ++sq[x];
                return true;
            };
            if (!(ok = issue_qk(0))) break;
            for (int j = 0; j < nb && ok; ++j) {
                if (j + 1 < nb && !(ok = issue_qk(j + 1))) break;
                const int st = (g0 + j) % kStages;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarVFull + st], ((g0 + j) / kStages) & 1))))
                    break;
                const int live = kv_end - j * kBN;            // rows of the block inside the causal range
                if (live < kBN) {
                    // rows past it may hold anything (NaN included): P is 0 there, 0 * NaN is not
                    uint8_t* vt = smem + kOffV + st * kKV;
                    for (int i = lane; i < (kBN - max(live, 0)) * 16; i += 32) {
                        const int r = max(live, 0) + (i >> 4), part = i & 15;
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
                        !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarOEmpty + x], (uo[x] - 1) & 1))))
                        break;
                    if (!(ok = __all_sync(0xffffffffu,
                                          mbar_wait(&bars[kBarPFull + x * 2 + (pv[x] & 1)], (pv[x] >> 1) & 1))))
                        break;
                    if (lane == 0) {
                        tc_fence_after();
                        const uint32_t pa = tmem + kColS + x * 128 + (pv[x] & 1) * kBN;   // P: 32 columns
                        const uint32_t vb = sbase + kOffV + st * kKV;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16_ts(tmem + kColO + x * 128, pa + kk * 8,
                                        umma_desc_sw128(vb + kk * 16 * 128, kKHalf, 1024), kIdescPV,
                                        (j > 0 || kk > 0) ? 1u : 0u);
                        umma_commit(&bars[kBarPvDone + x]);
                        if (j == nbx[x] - 1) umma_commit(&bars[kBarODone + x]);
                    }
                    __syncwarp();
                    ++pv[x];
                }
                if (!ok) break;
                if (lane == 0) umma_commit(&bars[kBarVEmpty + st]);
                __syncwarp();
            }
            gk = g0 + nb;
            for (int x = 0; x < 2; ++x)
                if (nbx[x] > 0) ++uo[x];
        }
        if (!ok) {
            if (lane == 0) {
                fail();
                umma_commit(&bars[kBarDrain]);
                (void)mbar_wait(&bars[kBarDrain], 0);            // MMAs issued so far have completed
            }
            __syncwarp();
        }
    } else if (warp < kWarpQ) {
        // ================================================= softmax + epilogue of tile x
        const int x = (warp - kWarpSoft0) >> 2;         // 0: tile A (warps 2..5), 1: tile B (warps 6..9)
        const int quad = warp & 3;                      // TMEM lanes 32*quad .. +31
        const int r = quad * 32 + lane;                 // this thread's row of the tile
        const int hh = r & 7;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
        const uint32_t col_s = kColS + x * 128;
        const uint32_t col_o = kColO + x * 128;
        const float sl2 = p.scale_log2;
        bool ok = true;
        int sq = 0;               // blocks processed (S/P buffer = sq & 1; also the PV count)
        int uo = 0;               // units finished (O phases)
        for (int k = 0; ok; ++k) {
            UnitDesc d;
            if (!(ok = __all_sync(0xffffffffu, wait_desc(k, d)))) break;
            free_desc(k);
            if (d.end) break;
            const int nbl = x ? d.nblk_b : d.nblk_a;
            if (nbl == 0) continue;                      // tile B of this unit has no live row
            const int t0 = d.t0 + x * kPos;
            const int tr = t0 + (r >> 3);                // this row's position (call index)
            const int prow = d.p0 + tr;                  // and its absolute position
            float m_ref = -INFINITY, e0 = 0.f, e1 = 0.f, r0 = 0.f, r1 = 0.f;
            // every tcgen05.ld/st is .sync.aligned and sits on warp-uniform control flow
            for (int j = 0; j < nbl; ++j, ++sq) {
                const int buf = sq & 1;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarSFull + x * 2 + buf], (sq >> 1) & 1)))) break;
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
                for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(v[i]));
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
                if (__any_sync(0xffffffffu, rescale)) {
                    // O must hold the PV of every earlier block of the unit (the one before this
                    // block may still run: QK of this block was issued before it)
                    if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarPvDone + x], (sq - 1) & 1)))) break;
                    tc_fence_after();
                    e0 *= alpha;
                    e1 *= alpha;
                    r0 *= alpha;
                    r1 *= alpha;
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        uint32_t o[16];
                        tmem_ld16(lane_base + col_o + q4 * 16, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st16(lane_base + col_o + q4 * 16, o);
                    }
                    tmem_wait_st();
                }
                // P = exp2(s * scale_log2 - mu) as bf16 pairs: keys 2c, 2c+1 in column c of the block's S
                // buffer (columns 0..31; the scores there are already in registers)
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    uint32_t pk[16];
#pragma unroll
                    for (int i = 0; i < 32; i += 2) {
                        const float s0 = fast_exp2(__uint_as_float(v[32 * h2 + i]) * sl2 - mu);
                        const float s1 = fast_exp2(__uint_as_float(v[32 * h2 + i + 1]) * sl2 - mu);
                        const __nv_bfloat162 pb = __floats2bfloat162_rn(s0, s1);
                        e0 += s0;
                        e1 += s1;
                        const float2 pf2 = __bfloat1622float2(pb);
                        r0 += pf2.x;
                        r1 += pf2.y;
                        pk[i >> 1] = *reinterpret_cast<const uint32_t*>(&pb);
                    }
                    tmem_st16(scol + 16 * h2, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bars[kBarPFull + x * 2 + buf]);
            }
            if (!ok) break;
            // ---- epilogue: O_x is complete once every MMA of the tile is
            if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarODone + x], uo & 1)))) break;
            ++uo;
            tc_fence_after();
            const float inv = 1.f / (r0 + r1);
            // bf16 row into the unit's finished Q tile, in the 128-byte-swizzled layout of the Q load
            uint8_t* stage = smem + kOffQ + (k & 1) * kQSlot + x * kQTile + r * 128;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                uint32_t o[32];
                tmem_ld32(lane_base + col_o + 32 * c4, o);
                tmem_wait_ld();
                if (c4 == 3) {
                    tc_fence_before();
                    mbar_arrive(&bars[kBarOEmpty + x]);            // the next unit may overwrite O_x
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint4 w;
                    w.x = pack_bf16x2(__uint_as_float(o[8 * q + 0]) * inv, __uint_as_float(o[8 * q + 1]) * inv);
                    w.y = pack_bf16x2(__uint_as_float(o[8 * q + 2]) * inv, __uint_as_float(o[8 * q + 3]) * inv);
                    w.z = pack_bf16x2(__uint_as_float(o[8 * q + 4]) * inv, __uint_as_float(o[8 * q + 5]) * inv);
                    w.w = pack_bf16x2(__uint_as_float(o[8 * q + 6]) * inv, __uint_as_float(o[8 * q + 7]) * inv);
                    const int chunk = (c4 & 1) * 4 + q;                   // 16-byte chunk within the half
                    *reinterpret_cast<uint4*>(stage + (c4 >> 1) * kQHalf + ((chunk ^ (r & 7)) << 4)) = w;
                }
            }
            fence_proxy_async_smem();                    // the TMA store reads the tile through the async proxy
            mbar_arrive(&bars[kBarStaged + x * 2 + (k & 1)]);
            if (tr < d.nn) {
                const int h = d.g * kGroup + hh;
                p.lse[d.l][(static_cast<size_t>(d.b) * p.Hq + h) * p.S + tr] = (m_ref + __log2f(e0 + e1)) * kLn2;
            }
        }
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
            !kv_tensor_map(&prm.vmap[i], cache_v[l], static_cast<long long>(B) * T, Hkv, 64, pf::kBN) ||
            !q_group_tensor_map(&prm.omap[i], o[l], static_cast<long long>(B) * S, Hq, 64, pf::kPos) ||
            !q_group_tensor_map(&prm.omap1[i], o[l], static_cast<long long>(B) * S, Hq, 64, 1))
            return ARK_ERR_CUDA;
        prm.lse[i] = lse[l];
    }
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
