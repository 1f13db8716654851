// Internal declarations shared by the libtpla.so translation units.
//
// Split-KV schedule (not on the TPLA pages; it is how one GPU keeps all SMs
// busy at small batch): the work of a call is a list of "units", one per
// (sequence b, shard s of the call, 64-token tile), ordered b-major, then
// shard, then tile.  Each unit has a cost weight, the same for all units of
// one sequence: the tcgen05 kernels spend more per tile on a sequence short
// enough for fp16 PV tiles (Plan::w_short against Plan::w_long).  With V the
// total weight and Vpos(u) the weight of the units before u, worker w (a CTA,
// or a CTA pair) takes the units whose Vpos lies in [v(w), v(w+1)),
// v(w) = floor(w * V / W): a contiguous unit range [lo(w), lo(w+1)).  Inside
// that range each run of one (b, s) is a "segment"; it leaves one partial
// result (normalised output rows + log2-sum-exp per head) in slot
//     W + b * gc + s         if the segment starts at tile 0 of (b, s),
//     w                      otherwise (it then starts the worker's range).
// The combine kernel rebuilds the same lists from seq_lens alone, so the host
// never needs the lengths and no kernel waits on another CTA.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/tpla.h"

namespace tpla {

constexpr int kPage = 64;            // tokens per cache page and per attention tile
constexpr int kMaxWorkers = 160;     // workspace is sized for this many split-KV workers
constexpr float kLog2e = 1.4426950408889634f;

// attention kernels (values of TPLA_OPT_LAST_ATTENTION_KERNEL)
constexpr int kKernelSimt = 1;       // CUDA cores, any supported shape
constexpr int kKernelSm100 = 2;      // tcgen05, L/g in {64, 128, 256}
constexpr int kKernelSm100Wide = 3;  // tcgen05, L/g = 512, a CTA pair per worker

// device status bits (tpla_check_device_status)
constexpr unsigned kStatusIndex = 1u;
constexpr unsigned kStatusTimeout = 2u;

struct Plan {
    int B, H, L, R, dv, g;
    int Ls;            // latent columns per shard (L / g)
    int gc;            // shards handled by this call (g, or 1 for a single-shard call)
    int shard0;        // first shard index of the call
    int max_pages, num_pages;
    int W;             // split-KV workers (a worker of the wide tcgen05 kernel is a CTA pair)
    int kernel;        // attention kernel: kKernelSimt, kKernelSm100 or kKernelSm100Wide
    int tile_tok;      // tokens per tile of the kKernelSm100 kernel: 64 or 128
    int w_long, w_short;   // split-KV cost weight of a unit of a sequence of >= / < short_below tokens
    int short_below;
    float scale_log2;  // softmax_scale * log2(e)
    unsigned* status;  // device status word (kStatus* bits)
};

struct Workspace {
    float* part_lse;   // [slots][H]
    float* part_o;     // [slots][H][Ls]
};

__host__ __device__ inline int num_slots(const Plan& p) { return p.W + p.B * p.gc; }

__host__ __device__ inline long long unit_lo(long long w, long long U, long long W) {
    return (w * U) / W;
}

// Worker that owns unit u (0 <= u < U): the largest w with lo(w) <= u.
__host__ __device__ inline int unit_worker(long long u, long long U, long long W) {
    return (int)(((u + 1) * W - 1) / U);
}

// Tokens of sequence b that are read: seq_lens[b] clamped to [0, 64 * max_pages];
// a clamp is a caller error and is recorded in the device status.
__device__ inline int effective_len(const int32_t* seq_lens, int b, int max_pages, unsigned* status) {
    int T = __ldg(seq_lens + b);
    int cap = max_pages * kPage;
    if (T < 0 || T > cap) {
        atomicOr(status, kStatusIndex);
        T = T < 0 ? 0 : cap;
    }
    return T;
}

__device__ inline int tiles_of_len(int T) { return (T + kPage - 1) / kPage; }

// Physical page of logical page `lp` of sequence b; -1 (recorded) if outside the cache.
__device__ inline int page_lookup(const int32_t* block_table, int b, int lp, int max_pages, int num_pages,
                                  unsigned* status) {
    int page = block_table ? __ldg(block_table + (size_t)b * max_pages + lp) : b * max_pages + lp;
    if (page < 0 || page >= num_pages) {
        atomicOr(status, kStatusIndex);
        return -1;
    }
    return page;
}

// Sum over b of gc * tiles(b), by one full warp (all 32 lanes call it).
__device__ inline long long warp_total_units(const int32_t* seq_lens, int B, int max_pages, int gc) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = 0; base < B; base += 32) {
        int b = base + lane;
        int n = 0;
        if (b < B) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
            n = tiles_of_len(T);
        }
        acc += n;
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc * gc;
}

// Cost weight of each unit of a sequence of T tokens (the split-KV schedule above).
__host__ __device__ inline int unit_weight(const Plan& p, int T) { return T < p.short_below ? p.w_short : p.w_long; }

// Sum over b of gc * tiles(b) * weight(b), by one full warp (all 32 lanes call it).
__device__ inline long long warp_total_weight(const int32_t* seq_lens, const Plan& p) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        if (b < p.B) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
            acc += (long long)tiles_of_len(T) * unit_weight(p, T);
        }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc * p.gc;
}

// The first unit (plain index) whose weighted start Vpos(u) is >= v, by one full warp; the total
// unit count when there is none.
__device__ inline long long warp_unit_at_weight(const int32_t* seq_lens, const Plan& p, long long v) {
    const int lane = threadIdx.x & 31;
    long long ubefore = 0, vbefore = 0;         // units and weight of sequences < base
    for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        long long n = 0;
        int c = 1;
        if (b < p.B) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
            n = (long long)tiles_of_len(T) * p.gc;
            c = unit_weight(p, T);
        }
        long long un = n, vn = n * c;           // inclusive scans over the 32 lanes
        for (int o = 1; o < 32; o <<= 1) {
            const long long a = __shfl_up_sync(0xffffffffu, un, o), bb = __shfl_up_sync(0xffffffffu, vn, o);
            if (lane >= o) { un += a; vn += bb; }
        }
        const long long vchunk = __shfl_sync(0xffffffffu, vn, 31);
        if (v < vbefore + vchunk) {
            // the first sequence whose weighted range ends past v holds the answer (or the next)
            const unsigned hit = __ballot_sync(0xffffffffu, b < p.B && v < vbefore + vn);
            const int src = __ffs(hit) - 1;
            const long long vs = vbefore + __shfl_sync(0xffffffffu, vn - n * c, src);   // its weighted start
            const long long us = ubefore + __shfl_sync(0xffffffffu, un - n, src);       // its first unit
            const int cs = __shfl_sync(0xffffffffu, c, src);
            const long long k = v <= vs ? 0 : (v - vs + cs - 1) / cs;                   // units before v's unit
            return us + k;
        }
        ubefore += __shfl_sync(0xffffffffu, un, 31);
        vbefore += vchunk;
    }
    return ubefore;
}

// Position of unit u in (b, s, tile) coordinates, found by one full warp.
// Returns b = B if u >= U.
struct UnitPos { int b, s, tile, ntiles, T; };

__device__ inline UnitPos warp_locate_unit(const int32_t* seq_lens, int B, int max_pages, int gc, long long u) {
    const int lane = threadIdx.x & 31;
    long long before = 0;                       // units of sequences < base
    for (int base = 0; base < B; base += 32) {
        int b = base + lane;
        int n = 0;
        if (b < B) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
            n = tiles_of_len(T) * gc;
        }
        long long incl = n;                     // inclusive scan over the 32 lanes
        for (int o = 1; o < 32; o <<= 1) {
            long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        long long chunk = __shfl_sync(0xffffffffu, incl, 31);
        if (u < before + chunk) {
            unsigned hit = __ballot_sync(0xffffffffu, b < B && u < before + incl);
            int src = __ffs(hit) - 1;
            long long excl = __shfl_sync(0xffffffffu, incl - n, src);
            int nb = __shfl_sync(0xffffffffu, n, src);
            UnitPos r;
            r.b = base + src;
            long long off = u - before - excl;
            int per = nb / gc;
            r.s = (int)(off / per);
            r.tile = (int)(off % per);
            r.ntiles = per;
            int T = __ldg(seq_lens + r.b);
            r.T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
            return r;
        }
        before += chunk;
    }
    UnitPos r; r.b = B; r.s = 0; r.tile = 0; r.ntiles = 0; r.T = 0;
    return r;
}

// Advance a unit position by one unit (scalar; skips empty sequences).
__device__ inline void advance_unit(UnitPos& p, const int32_t* seq_lens, int B, int max_pages, int gc) {
    if (++p.tile < p.ntiles) return;
    p.tile = 0;
    if (++p.s < gc) return;
    p.s = 0;
    for (;;) {
        if (++p.b >= B) { p.ntiles = 0; return; }
        int T = __ldg(seq_lens + p.b);
        T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
        p.T = T;
        p.ntiles = tiles_of_len(T);
        if (p.ntiles > 0) return;
    }
}

// Sets the dynamic shared-memory limit of `kern` once per device (a function
// attribute; repeating it on every launch only costs host time).
template <typename Kern>
inline cudaError_t set_smem_once(Kern kern, size_t bytes, unsigned long long* done_mask) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = 1ull << (dev & 63);
    if (__atomic_load_n(done_mask, __ATOMIC_ACQUIRE) & bit) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e == cudaSuccess) __atomic_fetch_or(done_mask, bit, __ATOMIC_RELEASE);
    return e;
}

// ---------------------------------------------------------------- programmatic dependent launch
//
// The kernels of a decode step are launched so that each may start while the previous kernel on the
// stream finishes (its prologue overlaps that kernel's tail).  pdl_wait() returns once the previous
// grid on the stream has completed and its writes are visible (at once when it was launched normally
// and has finished); pdl_trigger() lets the next grid launch.  Rules that keep this safe whatever
// the caller launches around the library:
//   * every CTA triggers only after its own wait has returned, so when a kernel starts, the kernel
//     two launches back has completed and everything it or earlier work wrote is visible;
//   * before its wait a kernel reads only data the immediately preceding kernel cannot write (the
//     combine, always preceded by the attention pass of the same call, stages W_UV and seq_lens),
//     and writes nothing to global memory.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launch `kern` on `stream` with programmatic stream serialisation allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// ---------------------------------------------------------------- launchers (one per .cu file)

cudaError_t launch_attention_simt(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                  const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                  const int32_t* block_table, const int32_t* seq_lens,
                                  Workspace ws, cudaStream_t stream);

// Returns cudaErrorNotSupported when the shape has no tcgen05 variant.
cudaError_t launch_attention_sm100(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                   const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                   const int32_t* block_table, const int32_t* seq_lens,
                                   Workspace ws, int wait_limit, int debug_stall, cudaStream_t stream);
bool sm100_supports(const Plan& p);

// Returns cudaErrorNotSupported when the shape is not L/g = 512 with R = 64.
cudaError_t launch_attention_sm100_wide(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                        const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                        const int32_t* block_table, const int32_t* seq_lens,
                                        Workspace ws, int wait_limit, int debug_stall, cudaStream_t stream);
bool sm100_wide_supports(const Plan& p);

cudaError_t launch_combine(const Plan& p, const int32_t* seq_lens, const __nv_bfloat16* w_uv,
                           float* out, Workspace ws, cudaStream_t stream);

// shard -1: every shard into the g-shard cache; otherwise shard `shard` alone into a one-shard cache
cudaError_t launch_append(const tpla_dims_t& d, int shard, const __nv_bfloat16* latent_raw,
                          const __nv_bfloat16* kpe_new, int transform, const float* R_dense,
                          const float* norm_weight, float eps, const int32_t* positions,
                          const int32_t* block_table, __nv_bfloat16* ckv, __nv_bfloat16* kpe,
                          unsigned* status, cudaStream_t stream);

}  // namespace tpla
