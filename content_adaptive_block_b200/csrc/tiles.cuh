// The tile list of one attention CTA: the union of two block lists (two CSR
// rows for a query tile, two CSC columns for a key tile), ascending, with a
// two-bit mark per entry telling which of the two halves it is live for.
#pragma once

#include "common.cuh"

namespace gsa {

constexpr int kListMaxBlocks = 2048;

struct TileList {
    int16_t* list;    // [kListMaxBlocks] block index per tile
    uint8_t* live;    // [kListMaxBlocks] bit 0: live for half 0, bit 1: for half 1
    uint32_t* bitsA;  // [kListMaxBlocks / 32]
    uint32_t* bitsB;  // [kListMaxBlocks / 32]
    int* count;       // number of entries
};

// Whole CTA.  lists: the CSR (or CSC) rows of this (sample, class), stored or
// implicit; a and b: the two rows (b < 0: none).  Ends with __syncthreads().
__device__ __forceinline__ void build_tile_list(const TileList& t, const ListRef& lists, int a, int b, int nblk) {
    const int nwords = (nblk + 31) >> 5;
    for (int k = threadIdx.x; k < nwords; k += blockDim.x) {
        t.bitsA[k] = 0u;
        t.bitsB[k] = 0u;
    }
    __syncthreads();
    lists.each(a, threadIdx.x, blockDim.x, [&](int j) { atomicOr(&t.bitsA[j >> 5], 1u << (j & 31)); });
    if (b >= 0) lists.each(b, threadIdx.x, blockDim.x, [&](int j) { atomicOr(&t.bitsB[j >> 5], 1u << (j & 31)); });
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int per = (nwords + 31) >> 5;
        const int w0 = lane * per, w1 = min(nwords, w0 + per);
        int cnt = 0;
        for (int k = w0; k < w1; ++k) cnt += __popc(t.bitsA[k] | t.bitsB[k]);
        int incl = cnt;
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = incl - cnt;
        for (int k = w0; k < w1; ++k) {
            const uint32_t ua = t.bitsA[k], ub = t.bitsB[k];
            uint32_t u = ua | ub;
            while (u) {
                const int bit = __ffs(u) - 1;
                u &= u - 1;
                t.list[pos] = static_cast<int16_t>(32 * k + bit);
                t.live[pos] = static_cast<uint8_t>(((ua >> bit) & 1u) | (((ub >> bit) & 1u) << 1));
                ++pos;
            }
        }
        if (lane == 31) *t.count = incl;
    }
    __syncthreads();
}

// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing `bar`'s transaction count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Store 64 fp32 values of one row as bf16 into a 128-byte-swizzled K-major
// tile (row r at r * 128 bytes, 16-byte chunk c at (c ^ (r % 8)) * 16).
__device__ __forceinline__ void store_row_sw128(uint8_t* tile, int r, const float* v) {
    uint8_t* row = tile + r * 128;
#pragma unroll
    for (int ch = 0; ch < 8; ++ch) {
        uint4 pk;
        pk.x = pack_bf16x2(v[8 * ch + 0], v[8 * ch + 1]);
        pk.y = pack_bf16x2(v[8 * ch + 2], v[8 * ch + 3]);
        pk.z = pack_bf16x2(v[8 * ch + 4], v[8 * ch + 5]);
        pk.w = pack_bf16x2(v[8 * ch + 6], v[8 * ch + 7]);
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) = pk;
    }
}

// Store 8 * nch fp32 values as bf16 into 16-byte chunks ch0 .. ch0+nch-1 of
// row r of a 128-byte-swizzled K-major tile.
__device__ __forceinline__ void store_cols_sw128(uint8_t* tile, int r, const float* v, int ch0, int nch) {
    uint8_t* row = tile + r * 128;
#pragma unroll
    for (int k = 0; k < nch; ++k) {
        const int ch = ch0 + k;
        uint4 pk;
        pk.x = pack_bf16x2(v[8 * k + 0], v[8 * k + 1]);
        pk.y = pack_bf16x2(v[8 * k + 2], v[8 * k + 3]);
        pk.z = pack_bf16x2(v[8 * k + 4], v[8 * k + 5]);
        pk.w = pack_bf16x2(v[8 * k + 6], v[8 * k + 7]);
        *reinterpret_cast<uint4*>(row + ((ch ^ (r & 7)) << 4)) = pk;
    }
}

// Store a row of 64 bf16 already packed in pairs (32 words) into a
// 128-byte-swizzled K-major tile.
__device__ __forceinline__ void store_packed_row_sw128(uint8_t* tile, int r, const uint32_t* pk) {
    uint8_t* row = tile + r * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (r & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
}

// Pairwise reductions (log-depth dependency chains instead of linear ones).
template <int N>
__device__ __forceinline__ float max_reduce(const float* v) {
    float t[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) t[i] = fmaxf(v[2 * i], v[2 * i + 1]);
#pragma unroll
    for (int w = N / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) t[i] = fmaxf(t[2 * i], t[2 * i + 1]);
    return t[0];
}

template <int N>
__device__ __forceinline__ float sum_reduce(const float* v) {
    float t[N / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) t[i] = v[2 * i] + v[2 * i + 1];
#pragma unroll
    for (int w = N / 4; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) t[i] = t[2 * i] + t[2 * i + 1];
    return t[0];
}

// Maximum of 32 values with three-input max: 17 instructions, depth 4.
__device__ __forceinline__ float max_reduce3_32(const float* v) {
    float t[11], u[4];
#pragma unroll
    for (int i = 0; i < 10; ++i) t[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    t[10] = fmaxf(v[30], v[31]);
#pragma unroll
    for (int i = 0; i < 3; ++i) u[i] = fmax3(t[3 * i], t[3 * i + 1], t[3 * i + 2]);
    u[3] = fmaxf(t[9], t[10]);
    return fmaxf(fmax3(u[0], u[1], u[2]), u[3]);
}

// Sum of 32 values as 16 packed pairs (v[2i], v[2i+1]): 16 instructions, depth 5.
__device__ __forceinline__ float sum_reduce2_32(const float* v) {
    uint64_t t[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) t[i] = f2_add(f2_pack(v[4 * i], v[4 * i + 1]), f2_pack(v[4 * i + 2], v[4 * i + 3]));
#pragma unroll
    for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) t[i] = f2_add(t[2 * i], t[2 * i + 1]);
    float lo, hi;
    f2_unpack(t[0], lo, hi);
    return lo + hi;
}

// 32 fp32 values times `mul` as bf16 to global memory (16-byte stores).
__device__ __forceinline__ void store_scaled_bf16(__nv_bfloat16* dst, const float* v, float mul) {
#pragma unroll
    for (int e = 0; e < 32; e += 8) {
        uint4 pk;
        pk.x = pack_bf16x2(v[e + 0] * mul, v[e + 1] * mul);
        pk.y = pack_bf16x2(v[e + 2] * mul, v[e + 3] * mul);
        pk.z = pack_bf16x2(v[e + 4] * mul, v[e + 5] * mul);
        pk.w = pack_bf16x2(v[e + 6] * mul, v[e + 7] * mul);
        *reinterpret_cast<uint4*>(dst + e) = pk;
    }
}

}  // namespace gsa
