// tma_host.h -- host-side encoding of TMA tensor maps over the KV cache, with
// a small cache so that repeated calls on the same buffers do not re-encode.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace ark {

// 3-D tiled map over a cache [B, T, Hkv, 128] bf16 viewed as
// (dim 0: 128 head-dim elements, dim 1: Hkv heads, dim 2: B*T rows), box
// (box_inner elements, 1 head, box_rows rows), 128-byte swizzle, zero fill
// out of bounds.  Returns false if the driver rejects it.
bool kv_tensor_map(CUtensorMap* out, const void* base, long long rows, int Hkv, int box_inner, int box_rows);

// 2-D tiled map over a row-major [rows, 128] bf16 matrix (row pitch 256 B),
// box (box_inner elements, box_rows rows), 128-byte swizzle.
// fp8 (one byte per element) cache, head-major [B][Hkv][T][128], 128-byte
// rows: dims (128, T, B*Hkv), box (128, box_rows, 1), 128-byte swizzle; a box
// is box_rows consecutive positions of one (request, KV head), contiguous in
// memory; positions past T read as zero.
bool kv8_tensor_map(CUtensorMap* out, const void* base, int B, int T, int Hkv, int box_rows);

// [rows][H][64] bf16 (heads of 64 dims): dims (64, H, rows), box (64, 1, box_rows),
// 128-byte swizzle.
bool hd64_tensor_map(CUtensorMap* out, const void* base, long long rows, int H, int box_rows);

// [rows][K] bf16, K contiguous (a K-major GEMM operand): dims (K, rows), box
// (64, box_rows), 128-byte swizzle.  K * 2 bytes must be a multiple of 16.
bool kmajor_tensor_map(CUtensorMap* out, const void* base, long long rows, int K, int box_rows);

bool rows_tensor_map(CUtensorMap* out, const void* base, long long rows, int box_inner, int box_rows);

// 4-D tiled map over q [B, S, Hq, 128] bf16 viewed as (dim 0: 128 head-dim
// elements, dim 1: 8 heads of a group, dim 2: Hq/8 groups, dim 3: B*S rows),
// box (box_inner, 8, 1, box_rows), 128-byte swizzle: one box lands as
// box_rows x 8 rows of box_inner elements, ordered (position, head).
bool q_group_tensor_map(CUtensorMap* out, const void* base, long long rows, int Hq, int box_inner, int box_rows);

}  // namespace ark
