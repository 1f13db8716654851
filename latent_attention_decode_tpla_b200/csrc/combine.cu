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
// One CTA = one head x a chunk of kBatchChunk sequences, so each W_UV_h
// slice is read once per chunk and reused for every sequence in it.
#include "tpla_internal.cuh"

namespace tpla {
namespace {

constexpr int kThreads = 256;
constexpr int kBatchChunk = 8;

// Units of all sequences before b (sum of gc * tiles), one full warp.
__device__ inline long long warp_units_before(const int32_t* seq_lens, int b_end, int max_pages, int gc) {
    const int lane = threadIdx.x & 31;
    long long acc = 0;
    for (int base = 0; base < b_end; base += 32) {
        int b = base + lane;
        if (b < b_end) {
            int T = __ldg(seq_lens + b);
            T = T < 0 ? 0 : (T > max_pages * kPage ? max_pages * kPage : T);
            acc += tiles_of_len(T);
        }
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    return acc * gc;
}

__global__ void __launch_bounds__(kThreads)
combine_kernel(Plan p, const int32_t* __restrict__ seq_lens, const __nv_bfloat16* __restrict__ w_uv,
               float* __restrict__ out, Workspace ws) {
    extern __shared__ __align__(16) float csm[];
    const int Lc = p.gc * p.Ls;                    // latent columns of this call
    float* o_lat = csm;                            // [kBatchChunk][Lc]
    float* red = csm + kBatchChunk * Lc;           // [groups][kBatchChunk][dv]
    __shared__ long long s_U, s_before;
    __shared__ int s_first_slot, s_wfirst, s_wlast;

    const int h = blockIdx.x;
    const int b0 = blockIdx.y * kBatchChunk;
    const int nb = min(kBatchChunk, p.B - b0);
    const int tid = threadIdx.x;

    if (tid < 32) {
        long long U = warp_total_units(seq_lens, p.B, p.max_pages, p.gc);
        long long before = warp_units_before(seq_lens, b0, p.max_pages, p.gc);
        if (tid == 0) { s_U = U; s_before = before; }
    }
    __syncthreads();
    const long long U = s_U;
    long long before = s_before;

    for (int bl = 0; bl < nb; ++bl) {
        const int b = b0 + bl;
        int T = __ldg(seq_lens + b);
        T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
        const int nt = tiles_of_len(T);
        for (int s = 0; s < p.gc; ++s) {
            float* dst = o_lat + bl * Lc + s * p.Ls;
            if (nt == 0) {
                for (int j = tid; j < p.Ls; j += kThreads) dst[j] = 0.f;
                continue;
            }
            const long long u0 = before + (long long)s * nt, u1 = u0 + nt - 1;
            __syncthreads();
            if (tid == 0) {
                int wf = unit_worker(u0, U, p.W);
                s_wfirst = wf;
                s_wlast = unit_worker(u1, U, p.W);
                s_first_slot = (unit_lo(wf, U, p.W) == u0) ? wf : p.W + b * p.gc + s;
            }
            __syncthreads();
            const int wf = s_wfirst, wl = s_wlast, fs = s_first_slot;
            // max log2-sum-exp over the segments of (b, s)
            float M = ws.part_lse[(size_t)fs * p.H + h];
            for (int wk = wf + 1; wk <= wl; ++wk)
                if (unit_lo(wk, U, p.W) < unit_lo(wk + 1, U, p.W))
                    M = fmaxf(M, ws.part_lse[(size_t)wk * p.H + h]);
            for (int j = tid; j < p.Ls; j += kThreads) {
                float wgt = exp2f(ws.part_lse[(size_t)fs * p.H + h] - M);
                float den = wgt;
                float num = wgt * ws.part_o[((size_t)fs * p.H + h) * p.Ls + j];
                for (int wk = wf + 1; wk <= wl; ++wk) {
                    if (unit_lo(wk, U, p.W) >= unit_lo(wk + 1, U, p.W)) continue;   // empty worker
                    float e = exp2f(ws.part_lse[(size_t)wk * p.H + h] - M);
                    den += e;
                    num = fmaf(e, ws.part_o[((size_t)wk * p.H + h) * p.Ls + j], num);
                }
                dst[j] = num / den;
            }
        }
        before += (long long)p.gc * nt;
    }
    __syncthreads();

    if (w_uv == nullptr) {
        for (int bl = 0; bl < nb; ++bl)
            for (int i = tid; i < Lc; i += kThreads)
                out[((size_t)(b0 + bl) * p.H + h) * Lc + i] = o_lat[bl * Lc + i];
        return;
    }
    // out[b, h, d] = sum_j o_lat[b][j] * W_UV[h][row(j)][d]
    const int groups = kThreads / p.dv;            // dv <= 256
    const int d = tid % p.dv, grp = tid / p.dv;
    const size_t row0 = (size_t)p.shard0 * p.Ls;   // first W_UV row of this call
    const __nv_bfloat16* wh = w_uv + ((size_t)h * p.L + row0) * p.dv;
    float acc[kBatchChunk];
#pragma unroll
    for (int bl = 0; bl < kBatchChunk; ++bl) acc[bl] = 0.f;
    if (grp < groups) {
        for (int j = grp; j < Lc; j += groups) {
            float wv = __bfloat162float(wh[(size_t)j * p.dv + d]);
#pragma unroll
            for (int bl = 0; bl < kBatchChunk; ++bl)
                if (bl < nb) acc[bl] = fmaf(o_lat[bl * Lc + j], wv, acc[bl]);
        }
#pragma unroll
        for (int bl = 0; bl < kBatchChunk; ++bl) red[(grp * kBatchChunk + bl) * p.dv + d] = acc[bl];
    }
    __syncthreads();
    for (int i = tid; i < nb * p.dv; i += kThreads) {
        int bl = i / p.dv, dd = i % p.dv;
        float sum = 0.f;
        for (int gi = 0; gi < groups; ++gi) sum += red[(gi * kBatchChunk + bl) * p.dv + dd];
        out[((size_t)(b0 + bl) * p.H + h) * p.dv + dd] = sum;
    }
}

}  // namespace

cudaError_t launch_combine(const Plan& p, const int32_t* seq_lens, const __nv_bfloat16* w_uv,
                           float* out, Workspace ws, cudaStream_t stream) {
    if (p.B == 0) return cudaSuccess;
    const int Lc = p.gc * p.Ls;
    const int groups = w_uv ? kThreads / p.dv : 0;
    const size_t smem = sizeof(float) * ((size_t)kBatchChunk * Lc + (size_t)groups * kBatchChunk * p.dv);
    cudaError_t e = cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(p.H, (p.B + kBatchChunk - 1) / kBatchChunk);
    combine_kernel<<<grid, kThreads, smem, stream>>>(p, seq_lens, w_uv, out, ws);
    return cudaGetLastError();
}

}  // namespace tpla
