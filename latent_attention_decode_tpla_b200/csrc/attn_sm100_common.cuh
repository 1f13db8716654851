// Pieces shared by the tcgen05 attention kernels (attn_sm100.cu, attn_sm100_wide.cu): the bounded
// pipeline wait, the tile cursor over a worker's unit range, the 128B-swizzle offset, and the
// host-side tensor maps.
#pragma once

#include "tpla_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda.h>
#include <mutex>

namespace tpla {
namespace sm100 {

// Bounded wait on an mbarrier phase shared by all roles of a CTA: a wait that runs out records
// TPLA_ERR_TIMEOUT in the device status word and raises the CTA's abort flag, so that every other
// role stops at its next wait instead of waiting for a partner that has given up.
struct Waiter {
    volatile int* abort;
    unsigned* status;
    uint64_t limit_cycles;

    // true when the phase of `parity` completed; false on abort or time-out
    // (the limit is counted in SM clock cycles: reading %globaltimer in the loop is slow)
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const long long t0 = clock64();
        for (;;) {
            if (mbar_try_wait(bar, parity)) return true;
            if (*abort) return false;
            if ((uint64_t)(clock64() - t0) > limit_cycles) {
                atomicOr(status, kStatusTimeout);
                *abort = 1;
                return false;
            }
        }
    }
};

// A tile: up to `maxp` consecutive units (pages) of one (sequence, shard) segment.
struct Tile {
    UnitPos pos;      // first unit of the tile
    long long u;      // its index in the unit order
    int npages;       // 1 .. maxp
    int maxp;         // pages per full tile
    bool begin, end;  // first / last tile of its segment
};

__device__ __forceinline__ Tile make_tile(const UnitPos& pos, long long u, long long lo, long long hi, int maxp) {
    Tile t;
    t.pos = pos;
    t.u = u;
    t.maxp = maxp;
    const long long left_seg = pos.ntiles - pos.tile;   // pages of this (b, s) from u on
    const long long left_rng = hi - u;                 // units of the worker from u on
    const long long left = left_seg < left_rng ? left_seg : left_rng;
    t.npages = left >= maxp ? maxp : (int)left;
    t.begin = u == lo || pos.tile == 0;
    t.end = t.npages == left;
    return t;
}

// the tile after `t`
__device__ __forceinline__ Tile next_tile(const Tile& t, const int32_t* seq_lens, const Plan& p, long long lo,
                                          long long hi) {
    UnitPos pos = t.pos;
    for (int k = 0; k < t.npages; ++k) advance_unit(pos, seq_lens, p.B, p.max_pages, p.gc);
    return make_tile(pos, t.u + t.npages, lo, hi, t.maxp);
}

// warp-collective: all lanes of the warp arrive through lane 0 after their prior writes
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// byte offset of 16-byte piece `c` of row `r` in a 128B-swizzled K-major operand (rows of 128 bytes)
__device__ __forceinline__ uint32_t sw128_offset(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// ------------------------------------------------------------------ PV number format of a tile
//
// PV multiplies P (rounded to 16 bits) by the bf16 latent tile, and one MMA never mixes types: P in
// bf16 (8 significant bits) costs about 1e-3 relative error on sequences of a few hundred tokens, P
// in fp16 (11 bits) about 1.5e-4, but an fp16 tile holds the latent values exactly only in fp16's
// normal range.  A short segment's tile therefore runs PV in fp16 with the latent values scaled by
// 2^e and P by 2^-e (the product is unchanged; both scalings are exact), e chosen from the tile's
// largest |value| so that it lands in [2^-10, 65280]: values 2^15 times smaller than the largest
// lose at most 2^-25 of it, and P (at most 2^8: the lazy rescale threshold) stays below 2^15.
// e is limited to [-7, 8], so this covers tiles whose largest |value| lies in [2^-18, 2^23); a
// tile outside that range, or holding inf or NaN, keeps bf16.
//
// `tmax` is the largest bf16 bit pattern of |value| over the tile's valid rows (for bf16, the
// unsigned order of these patterns is the order of the values).  Returns true for fp16 with shift e.
__device__ __forceinline__ bool pv_fp16_shift(uint32_t tmax, int& e) {
    const int E = (int)(tmax >> 7);                 // biased exponent of the largest value
    e = 0;
    if (tmax == 0u) return true;                    // all zero
    if (E >= 255) return false;                     // inf or NaN
    if (tmax > 0x477Fu) e = 142 - E;                // above 65280: shift down
    else if (tmax < 0x3A80u) e = 117 - E;           // below 2^-10: shift up
    return e >= -7 && e <= 8;
}

// two bf16 values (one 32-bit word) times 2^e -> fp16 (exact when the results are fp16 normals)
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_scaled(uint32_t v, float s) {
    return pack_f16x2(__uint_as_float(v << 16) * s, __uint_as_float(v & 0xFFFF0000u) * s);
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled, fetched from the driver once per process (the library links no driver
// library, so that it loads on machines without one)
inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// 3-D fp32 tensor map over the partial outputs [slots][H][cols] with a 32 x 32 x 1 box (32 columns of
// 32 rows of one slot) and 128-byte swizzle, for the TMA stores of the epilogues
inline bool make_map_o(CUtensorMap* m, void* base, uint64_t cols, uint64_t h, uint64_t slots) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cols, h, slots};
    cuuint64_t strides[2] = {cols * 4, h * cols * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over [rows][cols] with a 64 x 64 box and 128-byte swizzle
inline bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, 64};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace sm100
}  // namespace tpla
