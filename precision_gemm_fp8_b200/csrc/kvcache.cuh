// FP8 (E4M3) paged KV cache writer.
//
// "7B on an RTX 4060 with FP8": K/V stored in FP8 (half the cache);
// "C++ and FP8" §3.2: the cache is paged in blocks of tokens handed out by a
// central allocator and kept in FP8.  Layout (this library's reading):
// cache[block][kv head][slot][d], slot = position % block_size, the block of
// a position from a block table (position / block_size -> physical block);
// one scale per KV head (calibrated, e.g. pgf8_fp8_amax_accumulate per
// head); codes E4M3(RN(x / s_h)), saturating, with the quantisation's row
// division.
//
// Every 16-element chunk of a (token, head) row is one work item: a 128-bit
// load (f32 / f16 / bf16), 16 codes, one 16-byte store.  A block-table entry
// outside [0, num_blocks) is counted (once per token) and the token skipped:
// nothing is written outside the cache.
#pragma once

#include "quantize.cuh"

namespace pgf8 {

template <typename T>
__global__ void __launch_bounds__(kQuantThreads) kv_write_paged_kernel(
    const T *__restrict__ kv, int64_t ntok, int64_t H, int64_t D, int64_t ldkv, const float *__restrict__ scales,
    int64_t first_pos, int64_t B, const int32_t *__restrict__ block_table, int64_t num_blocks,
    uint8_t *__restrict__ cache, int32_t *__restrict__ bad_blocks)
{
    grid_launch_dependents();
    grid_dependency_wait();   // kv may come from the previous kernel (the K / V projection)
    const int64_t nch = D / 16;
    const int64_t total = ntok * H * nch;
    for (int64_t i = blockIdx.x * static_cast<int64_t>(kQuantThreads) + threadIdx.x; i < total;
         i += static_cast<int64_t>(gridDim.x) * kQuantThreads) {
        const int64_t c = i % nch, th = i / nch;
        const int64_t h = th % H, t = th / H;
        const int64_t pos = first_pos + t;
        const int64_t blk = block_table[pos / B];
        if (blk < 0 || blk >= num_blocks) {
            if (bad_blocks && h == 0 && c == 0)
                atomicAdd(bad_blocks, 1);
            continue;
        }
        Vec16<T> v;
        v.load(kv + t * ldkv + h * D + c * 16);
        const RowDivisor d(scales[h]);
        *reinterpret_cast<uint4 *>(cache + ((blk * H + h) * B + pos % B) * D + c * 16) = encode16(v.v, d);
    }
}

} // namespace pgf8
