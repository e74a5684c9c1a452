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
// Tiling: one CTA per (128 token rows, one head = 128 output features), two
// CTAs per SM.  The K dimension streams through a 3-stage ring of 64-wide
// chunks (x tile 16 KB, W tile 16 KB, 128-byte swizzle) loaded by TMA; one
// thread issues 4 MMAs of 128x128x16 per chunk into a 128-column TMEM
// accumulator.  When the tiles are too few to fill the GPU (a decode step: 20
// tiles of a few token rows, bound by streaming the 10.5 MB weight), K is split
// over a thread-block cluster of up to 8 CTAs: each sums its share of K, the
// others leave their fp32 partial tiles in shared memory, and the cluster's
// rank-0 CTA adds them in rank order over distributed shared memory (so the
// result does not depend on timing) before its epilogue.  Epilogue: 4 warps
// move the accumulator tile (one token row per thread) into shared memory; all
// 128 threads then take (row, 4 rotary pairs) items, the partners i and i + 64
// of a head being in the same row.  The projection value is the fp32
// accumulator plus the bias, added in double and rounded once to bf16; the
// rotation then works on
// that bf16 value exactly as the append kernel does, so the fused result is
// bit-identical to ark_attn_qkv_proj followed by ark_attn_append_rope.
#include "common.cuh"
#include "tma_host.h"

#include <mutex>

namespace ark {
namespace qp {

constexpr int kBM = 128;                 // token rows per tile (MMA M)
constexpr int kBN = 128;                 // output features per tile: one head (MMA N)
constexpr int kBK = 64;                  // K chunk: 64 bf16 = one 128-byte swizzle row
constexpr int kTileA = kBM * 128;        // 16 KB
constexpr int kTileB = kBN * 128;        // 16 KB
constexpr int kStageBytes = kTileA + kTileB;
constexpr int kThreads = 192;            // warp 0: TMA, warp 1: MMA, warps 2..5: epilogue

constexpr int kPartStride = 132;         // floats per row of a partial tile in shared memory (16-byte rows,
                                         // conflict-free float4 stores of 8 consecutive rows)

// Shared memory of a CTA with an S-stage ring: 3 stages (two CTAs per SM) when the tiles fill the
// GPU, 6 stages (one CTA per SM, more of a CTA's share of K in flight at once) when K is split.
template <int S>
struct Layout {
    static constexpr int kStages = S;
    static constexpr int kOffBar = S * kStageBytes;
    static constexpr int kBarFull = 0;                          // [S]
    static constexpr int kBarEmpty = kBarFull + S;              // [S]
    static constexpr int kBarDone = kBarEmpty + S;
    static constexpr int kNumBars = kBarDone + 1;
    static constexpr int kOffRows = kOffBar + kNumBars * 8;     // per tile row: int2 {destination / 8 or -1, pos}
    static constexpr int kOffBias = kOffRows + kBM * 8;         // this head's 128 bias values, fp32
    static constexpr int kOffTmemPtr = kOffBias + kBN * 4;
    static constexpr int kOffFlag = kOffTmemPtr + 8;
    static constexpr int kSmemBytes = kOffFlag + 8;
    static_assert(kBM * kPartStride * 4 <= kOffBar, "partial tile fits in the stage buffers");
};
constexpr int kStagesWide = 3;           // many tiles
constexpr int kStagesSplit = 6;          // K split over a cluster
constexpr int kMaxSplit = 8;             // portable cluster size
constexpr uint32_t kTmemCols = 128;

// kind::f16, bf16 x bf16 -> fp32, M = 128, N = 128, A and B K-major
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// The narrow form, for a few token rows (a decode step): the operands swap roles, so that the
// 128 output features of a head are the MMA's M and the token rows its N (nt = 16 .. 64).  A
// stage is then a 16 KB weight tile and a small x tile (room for XR rows), and the ring holds a
// cluster rank's whole share of K (hidden 2048 split 8 ways: 4 stages, two CTAs per SM): every
// weight copy is issued before the wait for the previous kernel, only the x copies after it,
// and the next layer's CTAs are resident beside this one's.  The split's partial tiles meet
// in `recv`: rank r owns token rows [r nt / split, (r+1) nt / split), and every rank pushes
// those rows of its fp32 tile into rank r's recv[rank] with st.async, which completes bytes on
// r's mbarrier -- no cluster-wide barrier sits between the MMAs and the epilogue.
constexpr int kNarrowMaxM = 64;
template <int NS, int XR>
struct NarrowLayout {
    static constexpr int kNStages = NS;
    static constexpr int kStage = kTileB + XR * 128;           // W tile + x tile of up to XR rows
    static constexpr int kOffRecv = NS * kStage;               // [split][128 features][nt / split] fp32
    static constexpr int kRecvBytes = XR * kBN * 4;
    static constexpr int kOffBar = kOffRecv + kRecvBytes;
    static constexpr int kBarFull = 0;                          // [NS]
    static constexpr int kBarEmpty = kBarFull + NS;             // [NS]
    static constexpr int kBarDone = kBarEmpty + NS;
    static constexpr int kBarRecv = kBarDone + 1;
    static constexpr int kNumBars = kBarRecv + 1;
    static constexpr int kOffRows = kOffBar + kNumBars * 8;     // per token row of this rank: int2
    static constexpr int kOffBias = kOffRows + XR * 8;
    static constexpr int kOffTmemPtr = kOffBias + kBN * 4;
    static constexpr int kOffFlag = kOffTmemPtr + 8;
    static constexpr int kSmemBytes = kOffFlag + 8;
    static_assert(kStage % 1024 == 0 && kTileB % 1024 == 0, "128-byte swizzled tiles start on 1 KB");
    static_assert(XR <= kNarrowMaxM && XR % 16 == 0, "x tile rows");
    static_assert(XR * kBN * 4 <= NS * kStage, "the summed rows fit over the stage buffers");
};
constexpr uint32_t kNarrowTmemCols = 64;
// kind::f16, bf16 x bf16 -> fp32, M = 128, N = n, A and B K-major
__host__ __device__ constexpr uint32_t idesc_m128(uint32_t n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

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
    int nt;                    // narrow form only: token rows per tile (MMA N), 16 .. 64
};

// Every thread of every CTA of the cluster, at the same program point.
__device__ __forceinline__ void cluster_sync_all() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16 bytes of another CTA's shared memory at this CTA's offset `local`.
__device__ __forceinline__ float4 ld_dsmem_f4(const void* local, uint32_t rank) {
    uint32_t raddr;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(raddr) : "r"(smem_u32(local)), "r"(rank));
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(raddr) : "memory");
    return v;
}

// 4 fp32 values (or one) into another CTA's shared memory at `raddr` (a shared::cluster
// address), completing their bytes on that CTA's mbarrier at `rbar`.
__device__ __forceinline__ void st_async_v4(uint32_t raddr, float a, float b, float c, float d, uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];"
                 :: "r"(raddr), "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar) : "memory");
}
__device__ __forceinline__ void st_async_f32(uint32_t raddr, float a, uint32_t rbar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 :: "r"(raddr), "r"(__float_as_uint(a)), "r"(rbar) : "memory");
}
__device__ __forceinline__ uint32_t map_rank(uint32_t local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}
// The narrow form's receive wait.  Every sender sends after at most one bounded wait of its
// own (kWaitLimitNs, in its epilogue), so a limit four times as long (on the global timer only)
// keeps a receiver from leaving while another rank may still write into its shared memory.
__device__ __forceinline__ bool mbar_wait_recv(uint64_t* bar, uint32_t parity) {
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t i = 0;; ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 63) == 63 && globaltimer_ns() - t0 > 4 * kWaitLimitNs) return false;
    }
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    __syncwarp();
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
    __syncwarp();
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// The plain projection of 8 output features of one token row: p = bf16(acc + bias), the sum in
// double and rounded once, stored as one 16-byte write at `dst`.
__device__ __forceinline__ void emit_plain8(uint16_t* dst, const float* sbias, int c8, float4 a0, float4 a1) {
    const float v[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double b0 = static_cast<double>(sbias[c8 + 2 * i]);
        const double b1 = static_cast<double>(sbias[c8 + 2 * i + 1]);
        w[i] = static_cast<uint32_t>(f64_to_bf16_rn(static_cast<double>(v[2 * i]) + b0)) |
               (static_cast<uint32_t>(f64_to_bf16_rn(static_cast<double>(v[2 * i + 1]) + b1)) << 16);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
}

// The fused form for one token row and rotary pairs 4g .. 4g+3 of one head: the projection
// value is the accumulator (lo: features 4g.., hi: features 64+4g..) plus the bias rounded once
// to bf16; q and k heads are then rotated exactly as by the append kernel (products exact in
// double, one rounding), v heads stored as they are.  info = {destination in 8-byte units, pos}.
// cs01, cs23: {cos, sin} of pairs 4g, 4g+1 and 4g+2, 4g+3 at the row's position (rope_pairs).
__device__ __forceinline__ void emit_rope_group(const Params& p, int head, int g, int2 info, const float* sbias,
                                                float4 lo, float4 hi, float4 cs01, float4 cs23) {
    uint16_t* base = head < p.Hq ? p.q : (head < p.Hq + p.Hkv ? p.cache_k : p.cache_v);
    uint16_t* dst = base + (static_cast<size_t>(info.x) << 2);
    const bool rotate = head < p.Hq + p.Hkv;
    const float al[4] = {lo.x, lo.y, lo.z, lo.w};
    const float ah[4] = {hi.x, hi.y, hi.z, hi.w};
    const float cc[4] = {cs01.x, cs01.z, cs23.x, cs23.z};
    const float ss[4] = {cs01.y, cs01.w, cs23.y, cs23.w};
    uint16_t yl[4], yh[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const double bl = static_cast<double>(sbias[4 * g + i]);
        const double bh = static_cast<double>(sbias[64 + 4 * g + i]);
        // the projection output (the Linear's bf16 value)
        const uint16_t xl = f64_to_bf16_rn(static_cast<double>(al[i]) + bl);
        const uint16_t xh = f64_to_bf16_rn(static_cast<double>(ah[i]) + bh);
        if (rotate) {
            const double a = bf16_bits_to_f64(xl);
            const double h = bf16_bits_to_f64(xh);
            const double c = static_cast<double>(cc[i]);
            const double sn = static_cast<double>(ss[i]);
            // both products are exact in double, so contraction cannot change the result
            yl[i] = f64_to_bf16_rn(a * c - h * sn);
            yh[i] = f64_to_bf16_rn(h * c + a * sn);
        } else {
            yl[i] = xl;
            yh[i] = xh;
        }
    }
    *reinterpret_cast<uint2*>(dst + 4 * g) =
        make_uint2(static_cast<uint32_t>(yl[0]) | (static_cast<uint32_t>(yl[1]) << 16),
                   static_cast<uint32_t>(yl[2]) | (static_cast<uint32_t>(yl[3]) << 16));
    *reinterpret_cast<uint2*>(dst + 64 + 4 * g) =
        make_uint2(static_cast<uint32_t>(yh[0]) | (static_cast<uint32_t>(yh[1]) << 16),
                   static_cast<uint32_t>(yh[2]) | (static_cast<uint32_t>(yh[3]) << 16));
}

// The rotary table entries of pairs 4g .. 4g+3 at position pos (zeros when the head is not
// rotated or pos is outside the table: such rows are not written).
__device__ __forceinline__ void rope_pairs(const Params& p, int head, int g, int pos, float4& cs01, float4& cs23) {
    if (head < p.Hq + p.Hkv && pos >= 0 && pos < p.T) {
        const float4* trow = reinterpret_cast<const float4*>(p.table + static_cast<size_t>(pos) * 64);
        cs01 = __ldg(trow + 2 * g);
        cs23 = __ldg(trow + 2 * g + 1);
    } else {
        cs01 = cs23 = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// Where token row m of a tile goes: {destination in 8-byte units or -1, position}; reports bad
// n_new / positions, and pulls the row's rotary table toward L2.
__device__ __forceinline__ int2 row_destination(const Params& p, int m, int head) {
    long long off = -1;
    int pos = 0;
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
            off = (static_cast<long long>(m) * p.Hq + head) * kHeadDim;
        } else if (head < p.Hq + p.Hkv) {
            off = ((static_cast<long long>(b) * p.T + pos) * p.Hkv + (head - p.Hq)) * kHeadDim;
        } else {
            off = ((static_cast<long long>(b) * p.T + pos) * p.Hkv + (head - p.Hq - p.Hkv)) * kHeadDim;
        }
        if (off >= 0 && head < p.Hq + p.Hkv) {
            const char* tr = reinterpret_cast<const char*>(p.table + static_cast<size_t>(pos) * 64);
#pragma unroll
            for (int i = 0; i < 4; ++i) asm volatile("prefetch.global.L2 [%0];" :: "l"(tr + 128 * i));
        }
    }
    // offsets are multiples of 128 elements; stored in 8-byte units they fit an int
    return make_int2(off < 0 ? -1 : static_cast<int>(off >> 2), pos);
}

}  // namespace qp

template <int S>
__global__ void __launch_bounds__(qp::kThreads, S <= 3 ? 2 : 1) qkv_proj_kernel(const __grid_constant__ qp::Params p) {
    using namespace qp;
    constexpr int kStages = Layout<S>::kStages;
    constexpr int kOffBar = Layout<S>::kOffBar;
    constexpr int kBarFull = Layout<S>::kBarFull;
    constexpr int kBarEmpty = Layout<S>::kBarEmpty;
    constexpr int kBarDone = Layout<S>::kBarDone;
    constexpr int kNumBars = Layout<S>::kNumBars;
    constexpr int kOffRows = Layout<S>::kOffRows;
    constexpr int kOffBias = Layout<S>::kOffBias;
    constexpr int kOffTmemPtr = Layout<S>::kOffTmemPtr;
    constexpr int kOffFlag = Layout<S>::kOffFlag;
    extern __shared__ __align__(1024) uint8_t smem[];
    // the next launch (the next layer's projection, launched with programmatic stream
    // serialisation) may start streaming its weights now; it reads its x and writes its
    // outputs only after griddepcontrol.wait, i.e. after this grid has completed
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int head = blockIdx.x;                 // output features 128*head .. +127
    const int m0 = blockIdx.y * kBM;
    // K split: this CTA sums chunks [c_begin, c_end); blockIdx.z is its rank in the cluster
    // (cluster dims (1, 1, gridDim.z)); no CTA returns early, every thread reaches the
    // cluster barriers below
    const int split = gridDim.z;
    const int rank = blockIdx.z;
    const int nk_all = p.K / kBK;
    const int c_begin = rank * nk_all / split;
    const int nk = (rank + 1) * nk_all / split - c_begin;
    const bool misaligned = (smem_u32(smem) & 1023u) != 0;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + kOffFlag);
    if (threadIdx.x == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], 1);
        *failed_flag = misaligned ? 1 : 0;
        if (misaligned) report(p.status, ARK_DEV_TIMEOUT);
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
            const int n_run = misaligned ? 0 : nk;
            // the weight tiles of the first stages do not depend on the previous kernel: they go first
            const int pre = min(n_run, kStages);
            for (int c = 0; c < pre; ++c) {
                mbar_arrive_expect_tx(&bars[kBarFull + c], kStageBytes);
                tma_load_2d(smem + c * kStageBytes + kTileA, &p.wmap, (c_begin + c) * kBK, head * kBN,
                            &bars[kBarFull + c]);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");    // x may be the previous kernel's output
            for (int c = 0; c < pre; ++c) {
                tma_load_2d(smem + c * kStageBytes, &p.xmap, (c_begin + c) * kBK, m0, &bars[kBarFull + c]);
                last = c;
            }
            for (int c = pre; c < n_run; ++c) {
                const int st = c % kStages;
                if (!(ok = mbar_wait(&bars[kBarEmpty + st], ((c / kStages) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[kBarFull + st], kStageBytes);
                const int kc = (c_begin + c) * kBK;
                tma_load_2d(smem + st * kStageBytes, &p.xmap, kc, m0, &bars[kBarFull + st]);
                tma_load_2d(smem + st * kStageBytes + kTileA, &p.wmap, kc, head * kBN, &bars[kBarFull + st]);
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
        for (int c = 0; c < (misaligned ? 0 : nk); ++c) {
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
    }

    // ================================================= epilogue
    // (1) every epilogue thread moves its TMEM row (a token row) into shared memory, over the
    // stage buffers, which are free once every MMA is done; (2) in a split cluster, rank 0 adds
    // the other ranks' tiles to its own, in rank order; (3) all 128 epilogue threads share the
    // live rows x 16 groups of 4 rotary pairs.  Every epilogue thread reaches every barrier.
    const int quad = warp & 3;               // TMEM lanes 32*quad .. +31
    const int r = quad * 32 + lane;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    float* part = reinterpret_cast<float*>(smem);          // [kBM][kPartStride] fp32
    const int rows = min(kBM, p.M - m0);                   // live token rows of this tile
    int2* rowinfo = reinterpret_cast<int2*>(smem + kOffRows);
    float* sbias = reinterpret_cast<float*>(smem + kOffBias);
    if (warp >= 2) {
        // the outputs may still be read by the previous kernel, and its pos0 / n_new / table writes
        // must be visible: nothing global is touched before it has completed
        asm volatile("griddepcontrol.wait;" ::: "memory");
        // while the MMAs run: where this thread's row goes (destination in 8-byte units, or -1),
        // its position, the head's bias, and the row's rotary table pulled toward L2
        {
            const int et = threadIdx.x - 64;
            sbias[et] = p.bias ? static_cast<float>(bf16_bits_to_f64(p.bias[head * kBN + et])) : 0.f;
            rowinfo[et] = (p.fused && et < rows && rank == 0) ? row_destination(p, m0 + et, head) : make_int2(-1, 0);
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBarDone], 0));
        tc_fence_after();
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        }
        for (int c16 = 0; c16 < kBN / 16; ++c16) {
            uint32_t a[16];
            tmem_ld16(lane_base + c16 * 16, a);
            tmem_wait_ld();
            if (ok && r < rows) {
                float4* d4 = reinterpret_cast<float4*>(part + r * kPartStride + c16 * 16);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    d4[i] = make_float4(__uint_as_float(a[4 * i]), __uint_as_float(a[4 * i + 1]),
                                        __uint_as_float(a[4 * i + 2]), __uint_as_float(a[4 * i + 3]));
            }
        }
    }
    if (split > 1) cluster_sync_all();       // the tiles of every rank are in place
    if (warp >= 2) {
        const int et = threadIdx.x - 64;     // 0 .. 127
        if (split > 1 && rank == 0) {
            // own + rank 1 + rank 2 + ..., each thread's remote loads issued before its adds
            const int items = rows * (kBN / 4);
            for (int it0 = et; it0 < items; it0 += 256) {
                // two pieces per pass: every remote load of both is in flight before the first add
                float* loc[2];
                float4 t[2][kMaxSplit - 1];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int it = min(it0 + 128 * u, items - 1);
                    loc[u] = part + (it / (kBN / 4)) * kPartStride + (it % (kBN / 4)) * 4;
#pragma unroll
                    for (int z = 1; z < kMaxSplit; ++z)
                        if (z < split) t[u][z - 1] = ld_dsmem_f4(loc[u], static_cast<uint32_t>(z));
                }
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    if (it0 + 128 * u >= items) continue;
                    float4 sum = *reinterpret_cast<const float4*>(loc[u]);
#pragma unroll
                    for (int z = 1; z < kMaxSplit; ++z)
                        if (z < split) {
                            sum.x += t[u][z - 1].x;
                            sum.y += t[u][z - 1].y;
                            sum.z += t[u][z - 1].z;
                            sum.w += t[u][z - 1].w;
                        }
                    *reinterpret_cast<float4*>(loc[u]) = sum;
                }
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");     // the tile's sums are complete
        const bool failed = *reinterpret_cast<volatile int*>(failed_flag) != 0;
        if (rank == 0 && !failed && !p.fused) {
            // p = bf16(acc + bias) -> out[m][128*head ..]: items of 8 columns
            for (int it = et; it < rows * (kBN / 8); it += 128) {
                const int row = it / (kBN / 8), c8 = (it % (kBN / 8)) * 8;
                const float* src = part + row * kPartStride + c8;
                emit_plain8(p.out + static_cast<size_t>(m0 + row) * p.N + head * kBN + c8, sbias, c8,
                            *reinterpret_cast<const float4*>(src), *reinterpret_cast<const float4*>(src + 4));
            }
        } else if (rank == 0 && !failed) {
            // items (row, group g of rotary pairs 4g .. 4g+3)
            for (int it = et; it < rows * 16; it += 128) {
                const int row = it >> 4, g = it & 15;
                const int2 info = rowinfo[row];
                if (info.x < 0) continue;                         // padded or out-of-range row: not written
                float4 cs01, cs23;
                rope_pairs(p, head, g, info.y, cs01, cs23);
                emit_rope_group(p, head, g, info, sbias,
                                *reinterpret_cast<const float4*>(part + row * kPartStride + 4 * g),
                                *reinterpret_cast<const float4*>(part + row * kPartStride + 64 + 4 * g), cs01, cs23);
            }
        }
    }
    if (split > 1) cluster_sync_all();       // rank 0 has read every other rank's tile: they may exit

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// The narrow form (see qp::NarrowLayout): D^T[128 features][nt tokens] = W_tile . x_tile^T in
// TMEM, one feature per TMEM lane.  Each epilogue thread sends its feature's values of rank r's
// token rows to rank r (its own rows by plain stores); rank r sums the split partials in rank
// order (rank 0's first, as the wide form adds), so the result does not depend on timing, and
// emits its rows with the wide form's arithmetic.  Every rank sends all its rows unconditionally
// (after bounded waits), so each owner's receive wait ends, and a CTA leaves only after the
// bytes sent to it have landed.
template <int NS, int XR>
__global__ void __launch_bounds__(qp::kThreads, NS <= 4 ? 2 : 1) qkv_proj_narrow_kernel(const __grid_constant__ qp::Params p) {
    using namespace qp;
    using Lay = NarrowLayout<NS, XR>;
    constexpr int kNStages = NS;
    constexpr int kStage = Lay::kStage;
    extern __shared__ __align__(1024) uint8_t smem[];
    // the next launch may start streaming its weights now (see qkv_proj_kernel)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int head = blockIdx.x;
    const int nt = p.nt;
    const int m0 = blockIdx.y * nt;
    const int split = gridDim.z;
    const int rank = blockIdx.z;
    const int nk_all = p.K / kBK;
    const int c_begin = rank * nk_all / split;
    const int nk = (rank + 1) * nk_all / split - c_begin;
    const int my_rows = nt / split;                    // token rows per rank (the host makes split divide nt)
    const uint32_t stage_tx = static_cast<uint32_t>(kTileB + nt * 128);
    const bool misaligned = (smem_u32(smem) & 1023u) != 0;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kOffBar);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + Lay::kOffTmemPtr);
    int* failed_flag = reinterpret_cast<int*>(smem + Lay::kOffFlag);
    float* recv = reinterpret_cast<float*>(smem + Lay::kOffRecv);
    if (threadIdx.x == 0) {
        for (int i = 0; i < Lay::kNumBars; ++i) mbar_init(&bars[i], 1);
        *failed_flag = misaligned ? 1 : 0;
        if (misaligned) report(p.status, ARK_DEV_TIMEOUT);
        // the other ranks' rows of this rank's tile: one arrival now, the bytes as they land
        mbar_arrive_expect_tx(&bars[Lay::kBarRecv], static_cast<uint32_t>((split - 1) * kBN * my_rows * 4));
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_ptr, kNarrowTmemCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // every rank's receive barrier is initialised before any rank sends (the wait comes before the sends)
    if (split > 1) cluster_arrive_relaxed();
    const uint32_t tmem = *tmem_ptr;
    const uint32_t sbase = smem_u32(smem);

    if (warp == 0) {
        // ================================================= TMA producer
        if (lane == 0) {
            int last = -1;
            bool ok = true;
            const int n_run = misaligned ? 0 : nk;
            // every weight tile that has a stage goes before the wait: they do not depend on the
            // previous kernel.  Each weight byte is read once per step: evict-first in L2, so that
            // the step's small operands (x, the rows the epilogue writes) stay there
            const uint64_t pol_w = l2_policy_evict_first();
            const int pre = min(n_run, kNStages);
            for (int c = 0; c < pre; ++c) {
                mbar_arrive_expect_tx(&bars[Lay::kBarFull + c], stage_tx);
                tma_load_2d_hint(smem + c * kStage, &p.wmap, (c_begin + c) * kBK, head * kBN, &bars[Lay::kBarFull + c],
                                 pol_w);
            }
            asm volatile("griddepcontrol.wait;" ::: "memory");    // x may be the previous kernel's output
            for (int c = 0; c < pre; ++c) {
                tma_load_2d(smem + c * kStage + kTileB, &p.xmap, (c_begin + c) * kBK, m0, &bars[Lay::kBarFull + c]);
                last = c;
            }
            for (int c = pre; c < n_run; ++c) {
                const int st = c % kNStages;
                if (!(ok = mbar_wait(&bars[Lay::kBarEmpty + st], ((c / kNStages) - 1) & 1))) break;
                mbar_arrive_expect_tx(&bars[Lay::kBarFull + st], stage_tx);
                const int kc = (c_begin + c) * kBK;
                tma_load_2d_hint(smem + st * kStage, &p.wmap, kc, head * kBN, &bars[Lay::kBarFull + st], pol_w);
                tma_load_2d(smem + st * kStage + kTileB, &p.xmap, kc, m0, &bars[Lay::kBarFull + st]);
                last = c;
            }
            if (!ok) {
                atomicExch(failed_flag, 1);
                report(p.status, ARK_DEV_TIMEOUT);
            }
            // the copies of the last stages have landed before the shared memory can go away
            for (int c = last - kNStages + 1; c <= last; ++c)
                if (c >= 0) (void)mbar_wait(&bars[Lay::kBarFull + c % kNStages], (c / kNStages) & 1);
        }
    } else if (warp == 1) {
        // ================================================= MMA issuer
        const uint32_t idesc = idesc_m128(static_cast<uint32_t>(nt));
        bool ok = true;
        if (nk <= kNStages) {
            // the whole share is in the ring: wait for all of it, then issue every MMA back to back
            for (int c = 0; c < (misaligned ? 0 : nk); ++c)
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[Lay::kBarFull + c], 0)))) break;
            if (ok && !misaligned && lane == 0) {
                tc_fence_after();
                for (int c = 0; c < nk; ++c) {
                    const uint32_t a = sbase + c * kStage;       // W tile: A, 128 features x 64 K
                    const uint32_t b = a + kTileB;                // x tile: B, nt tokens x 64 K
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem, umma_desc_sw128(a + kk * 32, 16, 1024), umma_desc_sw128(b + kk * 32, 16, 1024),
                                 idesc, (c > 0 || kk > 0) ? 1u : 0u);
                }
            }
            __syncwarp();
        } else {
            for (int c = 0; c < (misaligned ? 0 : nk); ++c) {
                const int st = c % kNStages;
                if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bars[Lay::kBarFull + st], (c / kNStages) & 1)))) break;
                if (lane == 0) {
                    tc_fence_after();
                    const uint32_t a = sbase + st * kStage;
                    const uint32_t b = a + kTileB;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        umma_f16(tmem, umma_desc_sw128(a + kk * 32, 16, 1024), umma_desc_sw128(b + kk * 32, 16, 1024),
                                 idesc, (c > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&bars[Lay::kBarEmpty + st]);
                }
                __syncwarp();
            }
        }
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        }
        __syncwarp();
        if (lane == 0) umma_commit(&bars[Lay::kBarDone]);     // also when the loop gave up
        __syncwarp();
    }

    // ================================================= epilogue
    const int quad = warp & 3;
    const int f = quad * 32 + lane;                        // this thread's feature (its TMEM lane)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const int rows = min(nt, p.M - m0);
    const int t0 = rank * my_rows;
    int2* rowinfo = reinterpret_cast<int2*>(smem + Lay::kOffRows);
    float* sbias = reinterpret_cast<float*>(smem + Lay::kOffBias);
    if (warp >= 2) {
        // nothing global is read before the previous kernel has completed (see qkv_proj_kernel)
        asm volatile("griddepcontrol.wait;" ::: "memory");
        {
            const int et = threadIdx.x - 64;
            sbias[et] = p.bias ? static_cast<float>(bf16_bits_to_f64(p.bias[head * kBN + et])) : 0.f;
            if (et < my_rows)
                rowinfo[et] = (p.fused && t0 + et < rows) ? row_destination(p, m0 + t0 + et, head)
                                                          : make_int2(-1, 0);
        }
        // the rotary table entries of this thread's first item (token row t0 + et / 16, group
        // et % 16), loaded while the MMAs run; any further items load theirs when they come
        float4 pre01 = make_float4(0.f, 0.f, 0.f, 0.f), pre23 = pre01;
        {
            const int et = threadIdx.x - 64;
            const int t = t0 + (et >> 4);
            if (p.fused && et < my_rows * 16 && t < rows) {
                const int m = m0 + t;
                const int b = m / p.S;
                rope_pairs(p, head, et & 15, __ldg(p.pos0 + b) + (m - b * p.S), pre01, pre23);
            }
        }
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[Lay::kBarDone], 0));
        tc_fence_after();
        if (!ok) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        }
        if (split > 1) cluster_wait();                     // every rank's receive barrier is set up
        // send: token t of this feature goes to recv[rank][f][t % my_rows] of rank t / my_rows
        const uint32_t my_slot = static_cast<uint32_t>((rank * kBN + f) * my_rows) * 4u;
        const uint32_t recv_local = smem_u32(recv) + my_slot;
        const uint32_t rbar_local = smem_u32(&bars[Lay::kBarRecv]);
        for (int c16 = 0; c16 < nt / 16; ++c16) {
            uint32_t a[16];
            tmem_ld16(lane_base + c16 * 16, a);
            tmem_wait_ld();
            if ((my_rows & 3) == 0) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int t = c16 * 16 + 4 * q4;
                    const int z = t / my_rows;
                    const uint32_t off = static_cast<uint32_t>(t - z * my_rows) * 4u;
                    const float v0 = __uint_as_float(a[4 * q4]), v1 = __uint_as_float(a[4 * q4 + 1]);
                    const float v2 = __uint_as_float(a[4 * q4 + 2]), v3 = __uint_as_float(a[4 * q4 + 3]);
                    if (z == rank)
                        *reinterpret_cast<float4*>(smem + Lay::kOffRecv + my_slot + off) = make_float4(v0, v1, v2, v3);
                    else
                        st_async_v4(map_rank(recv_local + off, static_cast<uint32_t>(z)), v0, v1, v2, v3,
                                    map_rank(rbar_local, static_cast<uint32_t>(z)));
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int t = c16 * 16 + i;
                    const int z = t / my_rows;
                    const uint32_t off = static_cast<uint32_t>(t - z * my_rows) * 4u;
                    if (z == rank)
                        *reinterpret_cast<float*>(smem + Lay::kOffRecv + my_slot + off) = __uint_as_float(a[i]);
                    else
                        st_async_f32(map_rank(recv_local + off, static_cast<uint32_t>(z)), __uint_as_float(a[i]),
                                     map_rank(rbar_local, static_cast<uint32_t>(z)));
                }
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");     // this rank's own rows are in recv
        bool got = true;
        if (split > 1) got = __all_sync(0xffffffffu, mbar_wait_recv(&bars[Lay::kBarRecv], 0));
        if (!got) {
            atomicExch(failed_flag, 1);
            if (lane == 0) report(p.status, ARK_DEV_TIMEOUT);
        }
        const bool failed = *reinterpret_cast<volatile int*>(failed_flag) != 0;
        // the split's partials of this thread's feature, summed for each of this rank's token rows
        // in rank order (rank 0's first), into sums[row][feature] over the stage buffers (free now
        // that every MMA has completed): 16-byte loads of 4 rows at a time, consecutive features
        // in consecutive threads, so the loads and stores are free of bank conflicts
        float* sums = reinterpret_cast<float*>(smem);
        if ((my_rows & 3) == 0) {
            for (int t4 = 0; t4 < my_rows; t4 += 4) {
                float4 acc = *reinterpret_cast<const float4*>(recv + f * my_rows + t4);
#pragma unroll
                for (int z = 1; z < kMaxSplit; ++z) {
                    if (z >= split) break;
                    const float4 v = *reinterpret_cast<const float4*>(recv + (z * kBN + f) * my_rows + t4);
                    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
                }
                sums[(t4 + 0) * kBN + f] = acc.x;
                sums[(t4 + 1) * kBN + f] = acc.y;
                sums[(t4 + 2) * kBN + f] = acc.z;
                sums[(t4 + 3) * kBN + f] = acc.w;
            }
        } else {
            for (int tl = 0; tl < my_rows; ++tl) {
                float acc = recv[f * my_rows + tl];
#pragma unroll
                for (int z = 1; z < kMaxSplit; ++z) {
                    if (z >= split) break;
                    acc += recv[(z * kBN + f) * my_rows + tl];
                }
                sums[tl * kBN + f] = acc;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");     // every row's sums are in place
        const int et = threadIdx.x - 64;
        // items (token row of this rank, group g): fused, features 4g.. and 64+4g..; plain, 8g .. 8g+7
        for (int it = et; it < my_rows * 16 && !failed; it += 128) {
            const int tl = it >> 4, g = it & 15;
            if (t0 + tl >= rows) continue;
            if (p.fused && rowinfo[tl].x < 0) continue;    // padded or out-of-range row: not written
            const float* row = sums + tl * kBN;
            const float4 sa = *reinterpret_cast<const float4*>(row + (p.fused ? 4 * g : 8 * g));
            const float4 sb = *reinterpret_cast<const float4*>(row + (p.fused ? 64 + 4 * g : 8 * g + 4));
            if (p.fused) {
                const int2 info = rowinfo[tl];
                if (it >= 128) rope_pairs(p, head, g, info.y, pre01, pre23);
                emit_rope_group(p, head, g, info, sbias, sa, sb, pre01, pre23);
            } else {
                emit_plain8(p.out + static_cast<size_t>(m0 + t0 + tl) * p.N + head * kBN + 8 * g, sbias, 8 * g, sa, sb);
            }
        }
    } else if (split > 1) {
        cluster_wait();                                    // (pairs with the arrival above)
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kNarrowTmemCols);
    }
}

}  // namespace ark

using namespace ark;

namespace {

bool qp_aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

std::mutex g_qp_mu;            // guards the per-device set-up below (first calls may come from several threads)
bool g_qp_attr[64];
int g_qp_sms[64];
int g_qp_clusters[64][4];    // clusters of 2, 4, 8 six-stage CTAs that can be resident at once (0: unknown)

template <int S>
ark_status launch_kernel(const qp::Params& prm, int M, int N, int split, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(N / qp::kBN, (M + qp::kBM - 1) / qp::kBM, split);
    cfg.blockDim = dim3(qp::kThreads);
    cfg.dynamicSmemBytes = qp::Layout<S>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(split);
    cfg.attrs = attr;
    cfg.numAttrs = split > 1 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, qkv_proj_kernel<S>, prm) != cudaSuccess) return ARK_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

// Clusters of `split` CTAs of `kernel` (with `smem` bytes) that can be resident at once, or -1.
int max_clusters(const void* kernel, int smem, int split) {
    cudaLaunchConfig_t occ = {};
    occ.gridDim = dim3(1, 1, split);
    occ.blockDim = dim3(qp::kThreads);
    occ.dynamicSmemBytes = smem;
    cudaLaunchAttribute ca[1];
    ca[0].id = cudaLaunchAttributeClusterDimension;
    ca[0].val.clusterDim.x = 1;
    ca[0].val.clusterDim.y = 1;
    ca[0].val.clusterDim.z = static_cast<unsigned>(split);
    occ.attrs = ca;
    occ.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &occ) != cudaSuccess) {
        (void)cudaGetLastError();
        return -1;
    }
    return n > 0 ? n : -1;
}

// The narrow form for M <= 64 token rows: nt = M rounded up to 16; K split 8 ways (4-stage
// ring, two CTAs per SM) when the hidden size allows it and the grid fits two CTAs per SM, else
// over the largest cluster whose clusters are all resident at once; the split divides nt.
template <int NS, int XR>
ark_status launch_narrow_ns(const qp::Params& prm, int tiles, int split, cudaStream_t stream) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(tiles, 1, split);
    cfg.blockDim = dim3(qp::kThreads);
    cfg.dynamicSmemBytes = qp::NarrowLayout<NS, XR>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = static_cast<unsigned>(split);
    cfg.attrs = attr;
    cfg.numAttrs = split > 1 ? 2 : 1;
    if (cudaLaunchKernelEx(&cfg, qkv_proj_narrow_kernel<NS, XR>, prm) != cudaSuccess) return ARK_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? ARK_OK : ARK_ERR_CUDA;
}

template <int NS, int XR>
cudaError_t narrow_smem_attr() {
    return cudaFuncSetAttribute(qkv_proj_narrow_kernel<NS, XR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                qp::NarrowLayout<NS, XR>::kSmemBytes);
}

// clusters of the narrow form resident at once (0: unknown), per device and x tile size (32 or
// 64 rows): of 2 and 4 CTAs of the deep-ring form, and of 8 CTAs of the 4-stage form
int g_qp_nclusters[64][2][4];
int g_qp_n8[64][2];

ark_status launch_narrow(qp::Params& prm, const void* x, const void* w, int M, int K, int N, int dev,
                         cudaStream_t stream) {
    const int nt = (M + 15) / 16 * 16;
    if (!kmajor_tensor_map(&prm.xmap, x, M, K, nt) || !kmajor_tensor_map(&prm.wmap, w, N, K, qp::kBN))
        return ARK_ERR_CUDA;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    prm.nt = nt;
    const int tiles = N / qp::kBN;
    const int nk = K / qp::kBK;
    const bool wide_x = nt > 32;
    int split = 1;
    if (nk % 8 == 0 && nk / 8 <= 4 && tiles * 8 <= 2 * g_qp_sms[dev]) {
        int& n8 = g_qp_n8[dev][wide_x ? 1 : 0];
        if (n8 == 0)
            n8 = wide_x ? max_clusters(reinterpret_cast<const void*>(qkv_proj_narrow_kernel<4, 64>),
                                       qp::NarrowLayout<4, 64>::kSmemBytes, 8)
                        : max_clusters(reinterpret_cast<const void*>(qkv_proj_narrow_kernel<4, 32>),
                                       qp::NarrowLayout<4, 32>::kSmemBytes, 8);
        if (n8 > 0) split = 8;
    }
    if (split == 1) {
        for (int cand = 2, ci = 0; cand <= 4; cand *= 2, ++ci) {
            if (nk % cand != 0) break;
            int& nc = g_qp_nclusters[dev][wide_x ? 1 : 0][ci];
            if (nc == 0)
                nc = wide_x ? max_clusters(reinterpret_cast<const void*>(qkv_proj_narrow_kernel<6, 64>),
                                           qp::NarrowLayout<6, 64>::kSmemBytes, cand)
                            : max_clusters(reinterpret_cast<const void*>(qkv_proj_narrow_kernel<8, 32>),
                                           qp::NarrowLayout<8, 32>::kSmemBytes, cand);
            if (nc < tiles) break;
            split = cand;
        }
    }
    const bool small = nk / split <= 4;
    if (wide_x)
        return small ? launch_narrow_ns<4, 64>(prm, tiles, split, stream) : launch_narrow_ns<6, 64>(prm, tiles, split, stream);
    return small ? launch_narrow_ns<4, 32>(prm, tiles, split, stream) : launch_narrow_ns<8, 32>(prm, tiles, split, stream);
}

ark_status launch_qkv(qp::Params& prm, const void* x, const void* w, int M, int K, int N, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return ARK_ERR_CUDA;
    std::lock_guard<std::mutex> lk(g_qp_mu);     // held through the split choice (it fills the cluster tables)
    if (!g_qp_attr[dev]) {
        if (cudaFuncSetAttribute(qkv_proj_kernel<qp::kStagesWide>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 qp::Layout<qp::kStagesWide>::kSmemBytes) != cudaSuccess ||
            cudaFuncSetAttribute(qkv_proj_kernel<qp::kStagesSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 qp::Layout<qp::kStagesSplit>::kSmemBytes) != cudaSuccess ||
            narrow_smem_attr<4, 32>() != cudaSuccess || narrow_smem_attr<8, 32>() != cudaSuccess ||
            narrow_smem_attr<4, 64>() != cudaSuccess || narrow_smem_attr<6, 64>() != cudaSuccess)
            return ARK_ERR_CUDA;
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return ARK_ERR_CUDA;
        g_qp_sms[dev] = sms;
        g_qp_attr[dev] = true;
    }
    if (M <= qp::kNarrowMaxM) return launch_narrow(prm, x, w, M, K, N, dev, stream);
    if (!kmajor_tensor_map(&prm.xmap, x, M, K, qp::kBM) || !kmajor_tensor_map(&prm.wmap, w, N, K, qp::kBN))
        return ARK_ERR_CUDA;
    prm.M = M;
    prm.K = K;
    prm.N = N;
    const int tiles = (N / qp::kBN) * ((M + qp::kBM - 1) / qp::kBM);
    // split K over a cluster of six-stage CTAs (one per SM) while the split CTAs fit on the SMs, every
    // cluster of the launch can be resident at once (one wave) and the chunks divide evenly
    int split = 1;
    const int nk = K / qp::kBK;
    for (int cand = 2, ci = 0; cand <= qp::kMaxSplit; cand *= 2, ++ci) {
        if (nk % cand != 0 || static_cast<long long>(tiles) * cand > g_qp_sms[dev]) break;
        if (g_qp_clusters[dev][ci] == 0)
            g_qp_clusters[dev][ci] = max_clusters(reinterpret_cast<const void*>(qkv_proj_kernel<qp::kStagesSplit>),
                                                  qp::Layout<qp::kStagesSplit>::kSmemBytes, cand);
        if (g_qp_clusters[dev][ci] < tiles) break;
        split = cand;
    }
    if (split > 1) return launch_kernel<qp::kStagesSplit>(prm, M, N, split, stream);
    return launch_kernel<qp::kStagesWide>(prm, M, N, 1, stream);
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
    // row destinations are kept as 32-bit counts of 8-byte units
    if (M >= (1LL << 31) || static_cast<long long>(B) * T >= (1LL << 31) || Hq + 2 * Hkv > 65535 ||
        (M + qp::kBM - 1) / qp::kBM > 65535 || M * Hq * (kHeadDim / 4) >= (1LL << 31) ||
        static_cast<long long>(B) * T * Hkv * (kHeadDim / 4) >= (1LL << 31))
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
