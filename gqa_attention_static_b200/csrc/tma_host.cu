// tma_host.cu -- TMA tensor-map encoding (driver entry point looked up through
// the runtime, so the library does not link libcuda directly) and its cache.
#include "tma_host.h"

#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <unordered_map>

namespace ark {
namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                              CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

struct Key {
    uintptr_t base;
    long long rows;
    int kind, hkv, inner, box_rows;
    bool operator==(const Key& o) const {
        return base == o.base && rows == o.rows && kind == o.kind && hkv == o.hkv && inner == o.inner &&
               box_rows == o.box_rows;
    }
};
struct KeyHash {
    size_t operator()(const Key& k) const {
        size_t h = std::hash<uintptr_t>()(k.base);
        h ^= std::hash<long long>()(k.rows) + 0x9e3779b97f4a7c15ull + (h << 6) + (h >> 2);
        h ^= static_cast<size_t>(k.kind * 131 + k.hkv * 17 + k.inner * 7 + k.box_rows) + (h << 6) + (h >> 2);
        return h;
    }
};

std::mutex g_mu;
std::unordered_map<Key, CUtensorMap, KeyHash>& cache() {
    static std::unordered_map<Key, CUtensorMap, KeyHash> m;
    return m;
}

bool cached_encode(const Key& key, CUtensorMap* out, cuuint32_t rank, const cuuint64_t* dims,
                   const cuuint64_t* strides, const cuuint32_t* box,
                   CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
    {
        std::lock_guard<std::mutex> lk(g_mu);
        auto it = cache().find(key);
        if (it != cache().end()) {
            std::memcpy(out, &it->second, sizeof(CUtensorMap));
            return true;
        }
    }
    EncodeFn fn = encode_fn();
    if (!fn) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    CUtensorMap m;
    if (fn(&m, dtype, rank, reinterpret_cast<void*>(key.base), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    std::memcpy(out, &m, sizeof(CUtensorMap));
    std::lock_guard<std::mutex> lk(g_mu);
    if (cache().size() > 4096) cache().clear();
    cache()[key] = m;
    return true;
}

}  // namespace

bool kv_tensor_map(CUtensorMap* out, const void* base, long long rows, int Hkv, int box_inner, int box_rows) {
    const Key key{reinterpret_cast<uintptr_t>(base), rows, 0, Hkv, box_inner, box_rows};
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(Hkv), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {256, static_cast<cuuint64_t>(Hkv) * 256};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_inner), 1, static_cast<cuuint32_t>(box_rows)};
    return cached_encode(key, out, 3, dims, strides, box);
}

bool kv8_tensor_map(CUtensorMap* out, const void* base, int B, int T, int Hkv, int box_rows) {
    // the key's `inner` slot holds T here: the map depends on how B*T splits into B and T
    const Key key{reinterpret_cast<uintptr_t>(base), static_cast<long long>(B) * T, 3, Hkv, T, box_rows};
    const cuuint64_t dims[3] = {128, static_cast<cuuint64_t>(T), static_cast<cuuint64_t>(B) * Hkv};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(T) * 128};
    const cuuint32_t box[3] = {128, static_cast<cuuint32_t>(box_rows), 1};
    return cached_encode(key, out, 3, dims, strides, box, CU_TENSOR_MAP_DATA_TYPE_UINT8);
}

bool hd64_tensor_map(CUtensorMap* out, const void* base, long long rows, int H, int box_rows) {
    const Key key{reinterpret_cast<uintptr_t>(base), rows, 4, H, 64, box_rows};
    const cuuint64_t dims[3] = {64, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[2] = {128, static_cast<cuuint64_t>(H) * 128};
    const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
    return cached_encode(key, out, 3, dims, strides, box);
}

bool q_group_tensor_map(CUtensorMap* out, const void* base, long long rows, int Hq, int box_inner, int box_rows) {
    const Key key{reinterpret_cast<uintptr_t>(base), rows, 2, Hq, box_inner, box_rows};
    const cuuint64_t dims[4] = {128, 8, static_cast<cuuint64_t>(Hq / 8), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[3] = {256, 2048, static_cast<cuuint64_t>(Hq) * 256};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), 8, 1, static_cast<cuuint32_t>(box_rows)};
    return cached_encode(key, out, 4, dims, strides, box);
}

bool kmajor_tensor_map(CUtensorMap* out, const void* base, long long rows, int K, int box_rows) {
    const Key key{reinterpret_cast<uintptr_t>(base), rows, 5, K, 64, box_rows};
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    return cached_encode(key, out, 2, dims, strides, box);
}

bool rows_tensor_map(CUtensorMap* out, const void* base, long long rows, int box_inner, int box_rows) {
    const Key key{reinterpret_cast<uintptr_t>(base), rows, 1, 0, box_inner, box_rows};
    const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {256};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_inner), static_cast<cuuint32_t>(box_rows)};
    return cached_encode(key, out, 2, dims, strides, box);
}

}  // namespace ark
