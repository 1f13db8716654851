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
// One CTA = one head x a group of up to kBatchGroup sequences (x a slice of
// the dv columns when W_UV_h does not fit in shared memory): the CTA first
// copies its W_UV_h rows into shared memory with wide independent loads,
// then merges and projects kBatchChunk sequences at a time from there.
#include "tpla_internal.cuh"

namespace tpla {
namespace {

constexpr int kThreads = 256;
constexpr int kBatchChunk = 8;                 // sequences projected together (accumulators per thread)
constexpr int kBatchGroup = 16;                // sequences per CTA
constexpr size_t kWSmemBudget = 128 * 1024;    // bytes of W_UV staged per CTA

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

// Merge of one (sequence, shard) by one warp: the slot list and softmax weights
// are built by the warp's lanes, then every lane accumulates its columns over
// all segments with independent vector loads.
__device__ void merge_one(const Plan& p, const Workspace& ws, int h, int b, int s, int nt, long long u0,
                          long long U, int* slots, float* wgts, float* dst) {
    const int lane = threadIdx.x & 31;
    if (nt == 0) {
        for (int j = lane * 4; j < p.Ls; j += 128) *reinterpret_cast<float4*>(dst + j) = make_float4(0, 0, 0, 0);
        return;
    }
    const long long u1 = u0 + nt - 1;
    const int wf = unit_worker(u0, U, p.W), wl = unit_worker(u1, U, p.W);
    if (lane == 0) slots[0] = unit_lo(wf, U, p.W) == u0 ? wf : p.W + b * p.gc + s;
    int n = 1;
    for (int base = wf + 1; base <= wl; base += 32) {
        const int wk = base + lane;
        const bool ok = wk <= wl && unit_lo(wk, U, p.W) < unit_lo(wk + 1, U, p.W);
        const unsigned m = __ballot_sync(0xffffffffu, ok);
        if (ok) slots[n + __popc(m & ((1u << lane) - 1u))] = wk;
        n += __popc(m);
    }
    __syncwarp();
    float M = -INFINITY;
    for (int k = lane; k < n; k += 32) M = fmaxf(M, __ldg(ws.part_lse + (size_t)slots[k] * p.H + h));
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float den = 0.f;
    for (int k = lane; k < n; k += 32) {
        const float e = exp2f(__ldg(ws.part_lse + (size_t)slots[k] * p.H + h) - M);
        wgts[k] = e;
        den += e;
    }
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    __syncwarp();
    const float inv = 1.0f / den;
    for (int j = lane * 4; j < p.Ls; j += 128) {
        float4 acc = make_float4(0, 0, 0, 0);
#pragma unroll 4
        for (int k = 0; k < n; ++k) {
            const float wk = wgts[k];
            const float4 v = __ldg(reinterpret_cast<const float4*>(ws.part_o + ((size_t)slots[k] * p.H + h) * p.Ls + j));
            acc.x = fmaf(wk, v.x, acc.x);
            acc.y = fmaf(wk, v.y, acc.y);
            acc.z = fmaf(wk, v.z, acc.z);
            acc.w = fmaf(wk, v.w, acc.w);
        }
        *reinterpret_cast<float4*>(dst + j) = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    }
    __syncwarp();
}

__global__ void __launch_bounds__(kThreads)
combine_kernel(Plan p, int dsub, const int32_t* __restrict__ seq_lens, const __nv_bfloat16* __restrict__ w_uv,
               float* __restrict__ out, Workspace ws) {
    extern __shared__ __align__(16) uint8_t csm_raw[];
    const int Lc = p.gc * p.Ls;                    // latent columns of this call
    const bool project = w_uv != nullptr;
    __nv_bfloat16* w_s = reinterpret_cast<__nv_bfloat16*>(csm_raw);                  // [Lc][dsub]
    float* o_lat = reinterpret_cast<float*>(csm_raw + (project ? (size_t)Lc * dsub * 2 : 0));  // [group][Lc]
    float* red = o_lat + kBatchGroup * Lc;                                           // [groups][chunk][dsub]
    constexpr int kWarps = kThreads / 32;
    __shared__ long long s_U;
    __shared__ long long s_start[kBatchGroup];
    __shared__ int s_nt[kBatchGroup];
    __shared__ int s_slot[kWarps][kMaxWorkers + 1];
    __shared__ float s_wgt[kWarps][kMaxWorkers + 1];

    const int h = blockIdx.x;
    const int d0 = blockIdx.z * dsub;
    const int bg0 = blockIdx.y * kBatchGroup;
    const int nbg = min(kBatchGroup, p.B - bg0);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (project) {
        // stage W_UV[h][row0 + j][d0 .. d0+dsub) for j < Lc: 16-byte pieces, all independent
        const size_t row0 = (size_t)p.shard0 * p.Ls;
        const int per_row = dsub / 8;
        const int n = Lc * per_row;
        const uint4* src = reinterpret_cast<const uint4*>(w_uv);
#pragma unroll 8
        for (int i = tid; i < n; i += kThreads) {
            const int j = i / per_row, c = i % per_row;
            reinterpret_cast<uint4*>(w_s)[i] =
                __ldg(src + (((size_t)h * p.L + row0 + j) * p.dv + d0) / 8 + c);
        }
    }
    if (warp == 0) {
        // units before each sequence of the group, and the total
        const long long U = warp_total_units(seq_lens, p.B, p.max_pages, p.gc);
        long long before = warp_units_before(seq_lens, bg0, p.max_pages, p.gc);
        if (lane == 0) {
            s_U = U;
            for (int bl = 0; bl < nbg; ++bl) {
                int T = __ldg(seq_lens + bg0 + bl);
                T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
                s_nt[bl] = tiles_of_len(T);
                s_start[bl] = before;
                before += (long long)p.gc * s_nt[bl];
            }
        }
    }
    __syncthreads();
    const long long U = s_U;
    // one warp per (sequence, shard) item
    for (int it = warp; it < nbg * p.gc; it += kWarps) {
        const int bl = it / p.gc, s = it % p.gc;
        merge_one(p, ws, h, bg0 + bl, s, s_nt[bl], s_start[bl] + (long long)s * s_nt[bl], U, s_slot[warp],
                  s_wgt[warp], o_lat + bl * Lc + s * p.Ls);
    }
    __syncthreads();

    if (!project) {
        for (int i = tid; i < nbg * Lc; i += kThreads)
            out[((size_t)(bg0 + i / Lc) * p.H + h) * Lc + i % Lc] = o_lat[i];
        return;
    }
    // out[b, h, d0 + d] = sum_j o_lat[b][j] * W_UV[h][row(j)][d0 + d]   (W from shared memory)
    const int groups = kThreads / dsub;
    const int d = tid % dsub, grp = tid / dsub;
    for (int c0 = 0; c0 < nbg; c0 += kBatchChunk) {
        const int nb = min(kBatchChunk, nbg - c0);
        if (grp < groups) {
            float acc[kBatchChunk];
#pragma unroll
            for (int bl = 0; bl < kBatchChunk; ++bl) acc[bl] = 0.f;
#pragma unroll 4
            for (int j = grp; j < Lc; j += groups) {
                const float wv = __bfloat162float(w_s[(size_t)j * dsub + d]);
#pragma unroll
                for (int bl = 0; bl < kBatchChunk; ++bl) acc[bl] = fmaf(o_lat[(c0 + bl) * Lc + j], wv, acc[bl]);
            }
#pragma unroll
            for (int bl = 0; bl < kBatchChunk; ++bl) red[(grp * kBatchChunk + bl) * dsub + d] = acc[bl];
        }
        __syncthreads();
        for (int i = tid; i < nb * dsub; i += kThreads) {
            const int bl = i / dsub, dd = i % dsub;
            float sum = 0.f;
            for (int gi = 0; gi < groups; ++gi) sum += red[(gi * kBatchChunk + bl) * dsub + dd];
            out[((size_t)(bg0 + c0 + bl) * p.H + h) * p.dv + d0 + dd] = sum;
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_combine(const Plan& p, const int32_t* seq_lens, const __nv_bfloat16* w_uv,
                           float* out, Workspace ws, cudaStream_t stream) {
    if (p.B == 0) return cudaSuccess;
    const int Lc = p.gc * p.Ls;
    // widest dv slice whose W_UV rows fit the shared-memory budget (dv % 8 == 0)
    int dsub = p.dv;
    while (w_uv && (size_t)Lc * dsub * 2 > kWSmemBudget && dsub % 16 == 0) dsub /= 2;
    const int groups = w_uv ? kThreads / dsub : 0;
    const size_t smem = (w_uv ? (size_t)Lc * dsub * 2 : 0) +
                        sizeof(float) * ((size_t)kBatchGroup * Lc + (size_t)groups * kBatchChunk * dsub);
    static unsigned long long attr_done = 0;
    constexpr size_t kMaxDyn = 200 * 1024;   // + static shared memory stays under 227 KB
    if (smem > kMaxDyn) return cudaErrorNotSupported;
    cudaError_t e = set_smem_once(combine_kernel, kMaxDyn, &attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(p.H, (p.B + kBatchGroup - 1) / kBatchGroup, w_uv ? p.dv / dsub : 1);
    combine_kernel<<<grid, kThreads, smem, stream>>>(p, dsub, seq_lens, w_uv, out, ws);
    return cudaGetLastError();
}

}  // namespace tpla
