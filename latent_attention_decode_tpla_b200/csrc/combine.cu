// Combine: split-KV merge, W_UV up-projection, and the sum over shards.
//
// For sequence b, head h and shard s the attention kernels left one partial
// (o_k, lse_k) per split-KV segment k (o_k normalised by its own softmax
// sum, lse_k = log2 of that sum plus the running max, in log2 units).  The
// exact per-shard output is the softmax-weighted merge
//     o_{b,h,s} = sum_k 2^(lse_k - M) o_k / sum_k 2^(lse_k - M),  M = max_k lse_k.
// Then (TPLA paper, Abstract: shard results are combined by an all-reduce,
// which on one GPU is this sum)
//     out_{b,h} = sum_s W_UV_h[s*Ls:(s+1)*Ls, :]^T o_{b,h,s}      (fp32)
// or, without W_UV, the shard outputs side by side.
//
// Two kernels, each a few dependent memory round trips deep:
//   merge_kernel    one CTA per (sequence, shard, 8 heads): the segment list
//                   of the (sequence, shard) is built once, then each warp
//                   merges one head with independent vector loads and writes
//                   o_{b,h,s} to the `merged` buffer (or straight to `out`
//                   when there is no W_UV);
//   project_kernel  one CTA per head (and dv slice): W_UV_h rows are copied
//                   asynchronously into shared memory and reused for every
//                   sequence of the batch.
#include "tpla_internal.cuh"

namespace tpla {
namespace {

constexpr int kMergeWarps = 8;                 // heads per merge CTA
constexpr int kProjThreads = 256;
constexpr int kProjChunk = 8;                  // sequences projected together (accumulators per thread)
constexpr size_t kWSmemBudget = 128 * 1024;    // bytes of W_UV staged per projection CTA

// Sum over sequences [b_begin, b_end) of gc * tiles, by one full warp.
__device__ inline long long warp_units_range(const int32_t* seq_lens, int b_begin, int b_end, int max_pages, int gc) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = b_begin; base < b_end; base += 32) {
        const int b = base + lane;
        if (b < b_end) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
            acc += tiles_of_len(T);
        }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc * gc;
}

__global__ void __launch_bounds__(kMergeWarps * 32)
merge_kernel(Plan p, const int32_t* __restrict__ seq_lens, Workspace ws, float* __restrict__ dst_base,
             int dst_cols) {
    __shared__ int s_slot[kMaxWorkers + 1];
    __shared__ int s_nseg;
    const int b = blockIdx.y / p.gc, s = blockIdx.y % p.gc;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int h = blockIdx.x * kMergeWarps + warp;

    int T = __ldg(seq_lens + b);
    T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
    const int nt = tiles_of_len(T);
    if (warp == 0 && nt > 0) {
        // segments of (b, s): the worker holding its first tile, then every later
        // non-empty worker up to the one holding its last tile
        const long long U = warp_units_range(seq_lens, 0, p.B, p.max_pages, p.gc);
        const long long u0 = warp_units_range(seq_lens, 0, b, p.max_pages, p.gc) + (long long)s * nt;
        const long long u1 = u0 + nt - 1;
        const int wf = unit_worker(u0, U, p.W), wl = unit_worker(u1, U, p.W);
        if (lane == 0) s_slot[0] = unit_lo(wf, U, p.W) == u0 ? wf : p.W + b * p.gc + s;
        int n = 1;
        for (int base = wf + 1; base <= wl; base += 32) {
            const int wk = base + lane;
            const bool ok = wk <= wl && unit_lo(wk, U, p.W) < unit_lo(wk + 1, U, p.W);
            const unsigned m = __ballot_sync(0xffffffffu, ok);
            if (ok) s_slot[n + __popc(m & ((1u << lane) - 1u))] = wk;
            n += __popc(m);
        }
        if (lane == 0) s_nseg = n;
    }
    __syncthreads();
    if (h >= p.H) return;
    float* dst = dst_base + ((size_t)b * p.H + h) * dst_cols + (size_t)s * p.Ls;
    if (nt == 0) {
        for (int j = lane * 4; j < p.Ls; j += 128) *reinterpret_cast<float4*>(dst + j) = make_float4(0, 0, 0, 0);
        return;
    }
    const int n = s_nseg;
    // softmax weights of the segments for this head
    float M = -INFINITY;
    for (int k = lane; k < n; k += 32) M = fmaxf(M, __ldg(ws.part_lse + (size_t)s_slot[k] * p.H + h));
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int k = lane; k < n; k += 32) den += exp2f(__ldg(ws.part_lse + (size_t)s_slot[k] * p.H + h) - M);
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = 1.0f / den;
    for (int j = lane * 4; j < p.Ls; j += 128) {
        float4 acc = make_float4(0, 0, 0, 0);
#pragma unroll 8
        for (int k = 0; k < n; ++k) {
            const size_t slot = (size_t)s_slot[k];
            const float wk = exp2f(__ldg(ws.part_lse + slot * p.H + h) - M) * inv;
            const float4 v = __ldg(reinterpret_cast<const float4*>(ws.part_o + (slot * p.H + h) * p.Ls + j));
            acc.x = fmaf(wk, v.x, acc.x);
            acc.y = fmaf(wk, v.y, acc.y);
            acc.z = fmaf(wk, v.z, acc.z);
            acc.w = fmaf(wk, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(dst + j) = acc;
    }
}

__global__ void __launch_bounds__(kProjThreads)
project_kernel(Plan p, int dsub, const __nv_bfloat16* __restrict__ w_uv, const float* __restrict__ merged,
               float* __restrict__ out) {
    extern __shared__ __align__(16) uint8_t psm[];
    const int Lc = p.gc * p.Ls;
    __nv_bfloat16* w_s = reinterpret_cast<__nv_bfloat16*>(psm);                    // [Lc][dsub]
    float* o_s = reinterpret_cast<float*>(psm + (size_t)Lc * dsub * 2);            // [chunk][Lc]
    float* red = o_s + kProjChunk * Lc;                                             // [groups][chunk][dsub]
    const int h = blockIdx.x;
    const int d0 = blockIdx.y * dsub;
    const int tid = threadIdx.x;

    {   // W_UV[h][row0 + j][d0 .. d0+dsub) for j < Lc, 16-byte asynchronous copies
        const size_t row0 = (size_t)p.shard0 * p.Ls;
        const int per_row = dsub / 8;
        const int n = Lc * per_row;
        const uint4* src = reinterpret_cast<const uint4*>(w_uv);
        for (int i = tid; i < n; i += kProjThreads) {
            const int j = i / per_row, c = i % per_row;
            const uint4* g = src + (((size_t)h * p.L + row0 + j) * p.dv + d0) / 8 + c;
            const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(reinterpret_cast<uint4*>(w_s) + i));
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(g) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    }
    const int groups = kProjThreads / dsub;
    const int d = tid % dsub, grp = tid / dsub;
    for (int c0 = 0; c0 < p.B; c0 += kProjChunk) {
        const int nb = min(kProjChunk, p.B - c0);
        // merged rows of this head for the chunk of sequences (rows past nb are zero)
        for (int i = tid; i < kProjChunk * Lc / 4; i += kProjThreads) {
            const int bl = i / (Lc / 4), j4 = i % (Lc / 4);
            reinterpret_cast<float4*>(o_s)[i] =
                bl < nb ? __ldg(reinterpret_cast<const float4*>(merged + ((size_t)(c0 + bl) * p.H + h) * Lc) + j4)
                        : make_float4(0, 0, 0, 0);
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        if (grp < groups) {
            float acc[kProjChunk];
#pragma unroll
            for (int bl = 0; bl < kProjChunk; ++bl) acc[bl] = 0.f;
#pragma unroll 4
            for (int j = grp; j < Lc; j += groups) {
                const float wv = __bfloat162float(w_s[(size_t)j * dsub + d]);
#pragma unroll
                for (int bl = 0; bl < kProjChunk; ++bl) acc[bl] = fmaf(o_s[bl * Lc + j], wv, acc[bl]);
            }
#pragma unroll
            for (int bl = 0; bl < kProjChunk; ++bl) red[(grp * kProjChunk + bl) * dsub + d] = acc[bl];
        }
        __syncthreads();
        for (int i = tid; i < nb * dsub; i += kProjThreads) {
            const int bl = i / dsub, dd = i % dsub;
            float sum = 0.f;
            for (int gi = 0; gi < groups; ++gi) sum += red[(gi * kProjChunk + bl) * dsub + dd];
            out[((size_t)(c0 + bl) * p.H + h) * p.dv + d0 + dd] = sum;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_combine(const Plan& p, const int32_t* seq_lens, const __nv_bfloat16* w_uv,
                           float* out, Workspace ws, cudaStream_t stream) {
    if (p.B == 0) return cudaSuccess;
    const int Lc = p.gc * p.Ls;
    dim3 mgrid((p.H + kMergeWarps - 1) / kMergeWarps, p.B * p.gc);
    if (w_uv == nullptr) {
        merge_kernel<<<mgrid, kMergeWarps * 32, 0, stream>>>(p, seq_lens, ws, out, Lc);
        return cudaGetLastError();
    }
    merge_kernel<<<mgrid, kMergeWarps * 32, 0, stream>>>(p, seq_lens, ws, ws.merged, Lc);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // widest dv slice whose W_UV rows fit the shared-memory budget (dv % 8 == 0)
    int dsub = p.dv;
    while ((size_t)Lc * dsub * 2 > kWSmemBudget && dsub % 16 == 0) dsub /= 2;
    const int groups = kProjThreads / dsub;
    const size_t smem = (size_t)Lc * dsub * 2 + sizeof(float) * ((size_t)kProjChunk * Lc + (size_t)groups * kProjChunk * dsub);
    constexpr size_t kMaxDyn = 200 * 1024;
    if (smem > kMaxDyn) return cudaErrorNotSupported;
    static unsigned long long attr_done = 0;
    e = set_smem_once(project_kernel, kMaxDyn, &attr_done);
    if (e != cudaSuccess) return e;
    dim3 pgrid(p.H, p.dv / dsub);
    project_kernel<<<pgrid, kProjThreads, smem, stream>>>(p, dsub, w_uv, ws.merged, out);
    return cudaGetLastError();
}

}  // namespace tpla
