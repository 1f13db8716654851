// Cache append: orthogonal reparameterisation, sliced RMSNorm, paged store.
//
// edgentiq blog, "How TPLA Works: Smart Slicing and Reparameterization":
// an orthogonal transform (Hadamard or PCA) is applied to the latent before
// it is cut into shards, so that the RMSNorm each shard computes on its own
// slice stays close to the global one.  Per new token b:
//     y   = R x_b                      (Hadamard: fast Walsh-Hadamard transform, 1/sqrt(L))
//     c_s = y_s / sqrt(mean(y_s^2) + eps)  [* w_s]   for every shard s
// rounded to bf16 (round to nearest even) and written to
// ckv[page][s][slot][:], with k_pe copied to kpe[page][slot][:].
// One CTA per new token; this is latency-bound (one token per sequence).
#include "tpla_internal.cuh"

namespace tpla {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxL = 1024;

__global__ void __launch_bounds__(kThreads)
append_kernel(int L, int R, int g, int max_pages, int num_pages,
              const __nv_bfloat16* __restrict__ latent_raw, const __nv_bfloat16* __restrict__ kpe_new,
              int transform, const float* __restrict__ R_dense, const float* __restrict__ norm_weight,
              float eps, const int32_t* __restrict__ positions, const int32_t* __restrict__ block_table,
              __nv_bfloat16* __restrict__ ckv, __nv_bfloat16* __restrict__ kpe, unsigned* status) {
    __shared__ float x[kMaxL];
    __shared__ float y[kMaxL];
    __shared__ float part[kMaxL / 32];
    __shared__ float inv_rms[8];
    const int b = blockIdx.x, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int Ls = L / g;

    const int pos = __ldg(positions + b);
    if (pos < 0 || pos >= max_pages * kPage) {
        if (tid == 0) atomicOr(status, kStatusIndex);
        return;
    }
    const int page = page_lookup(block_table, b, pos / kPage, max_pages, num_pages, status);
    if (page < 0) return;
    const int slot = pos % kPage;

    for (int i = tid; i < L; i += kThreads) x[i] = __bfloat162float(latent_raw[(size_t)b * L + i]);
    __syncthreads();

    if (transform == TPLA_TRANSFORM_HADAMARD) {
        // in-place radix-2 butterflies over L = 2^k points (Sylvester order), then 1/sqrt(L)
        for (int i = tid; i < L; i += kThreads) y[i] = x[i];
        __syncthreads();
        for (int hlen = 1; hlen < L; hlen <<= 1) {
            for (int k = tid; k < L / 2; k += kThreads) {
                int i = (k / hlen) * 2 * hlen + (k % hlen);
                float a = y[i], c = y[i + hlen];
                y[i] = a + c;
                y[i + hlen] = a - c;
            }
            __syncthreads();
        }
        const float sc = 1.0f / sqrtf((float)L);
        for (int i = tid; i < L; i += kThreads) y[i] *= sc;
    } else if (transform == TPLA_TRANSFORM_DENSE) {
        // y_i = sum_j R[i][j] x_j : one warp per output row, coalesced over j
        for (int i = warp; i < L; i += kThreads / 32) {
            const float* row = R_dense + (size_t)i * L;
            float acc = 0.f;
            for (int j = lane; j < L; j += 32) acc = fmaf(__ldg(row + j), x[j], acc);
            for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
            if (lane == 0) y[i] = acc;
        }
    } else {
        for (int i = tid; i < L; i += kThreads) y[i] = x[i];
    }
    __syncthreads();

    // sum of squares per 32-element chunk, then per shard
    for (int c = warp; c < L / 32; c += kThreads / 32) {
        float v = y[c * 32 + lane];
        float ss = v * v;
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) part[c] = ss;
    }
    __syncthreads();
    if (tid < g) {
        float ss = 0.f;
        for (int c = tid * (Ls / 32); c < (tid + 1) * (Ls / 32); ++c) ss += part[c];
        inv_rms[tid] = 1.0f / sqrtf(ss / (float)Ls + eps);
    }
    __syncthreads();

    for (int i = tid; i < L; i += kThreads) {
        int s = i / Ls, j = i % Ls;
        float v = y[i] * inv_rms[s];
        if (norm_weight) v *= __ldg(norm_weight + i);
        ckv[(((size_t)page * g + s) * kPage + slot) * Ls + j] = __float2bfloat16_rn(v);
    }
    for (int r = tid; r < R; r += kThreads)
        kpe[((size_t)page * kPage + slot) * R + r] = kpe_new[(size_t)b * R + r];
}

}  // namespace

cudaError_t launch_append(const tpla_dims_t& d, const __nv_bfloat16* latent_raw,
                          const __nv_bfloat16* kpe_new, int transform, const float* R_dense,
                          const float* norm_weight, float eps, const int32_t* positions,
                          const int32_t* block_table, __nv_bfloat16* ckv, __nv_bfloat16* kpe,
                          unsigned* status, cudaStream_t stream) {
    if (d.B == 0) return cudaSuccess;
    if (d.L > kMaxL) return cudaErrorNotSupported;
    append_kernel<<<d.B, kThreads, 0, stream>>>(d.L, d.R, d.g, d.max_pages_per_seq, d.num_pages,
                                                latent_raw, kpe_new, transform, R_dense, norm_weight,
                                                eps, positions, block_table, ckv, kpe, status);
    return cudaGetLastError();
}

}  // namespace tpla
