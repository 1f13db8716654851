// Cache append: orthogonal reparameterisation, sliced RMSNorm, paged store.
//
// edgentiq blog, "How TPLA Works: Smart Slicing and Reparameterization":
// an orthogonal transform (Hadamard or PCA) is applied to the latent before
// it is cut into shards, so that the RMSNorm each shard computes on its own
// slice stays close to the global one.  Per new token b:
//     y   = R x_b                      (Hadamard: fast Walsh-Hadamard transform, 1/sqrt(L);
//                                       block Hadamard: the same butterflies restricted to each
//                                       shard's L/g columns, 1/sqrt(L/g))
//     c_s = y_s / sqrt(mean(y_s^2) + eps)  [* w_s]   for every shard s
// rounded to bf16 (round to nearest even) and written to
// ckv[page][s][slot][:], with k_pe copied to kpe[page][slot][:].
// One CTA per (new token, shard of the call): the Hadamard transform is computed whole in
// every shard's CTA (it mixes all L inputs and costs L log L adds), the dense
// transform only for the shard's L/g rows, four rows per warp at a time so that
// many loads of R are in flight.  Each CTA normalises and stores its own
// slice; the first CTA of the token also copies k_pe.  A single-shard call (one tensor-parallel
// rank) computes shard s only and writes it into a cache that holds that shard alone.  Latency-bound: one token per
// sequence.
#include "tpla_internal.cuh"

namespace tpla {
namespace {

constexpr int kThreads = 512;
constexpr int kMaxL = 1024;

__global__ void __launch_bounds__(kThreads)
append_kernel(int L, int R, int g, int shard0, int g_out, int max_pages, int num_pages,
              const __nv_bfloat16* __restrict__ latent_raw, const __nv_bfloat16* __restrict__ kpe_new,
              int transform, const float* __restrict__ R_dense, const float* __restrict__ norm_weight,
              float eps, const int32_t* __restrict__ positions, const int32_t* __restrict__ block_table,
              __nv_bfloat16* __restrict__ ckv, __nv_bfloat16* __restrict__ kpe, unsigned* status) {
    __shared__ float x[kMaxL];
    __shared__ float y[kMaxL];
    __shared__ float part[kMaxL / 32];
    __shared__ float inv_rms[8];
    // shard sh of the transformed latent goes to shard slot blockIdx.y of a cache laid out with g_out
    // shards per page (g_out == g: all shards; g_out == 1: one tensor-parallel rank's cache)
    const int b = blockIdx.x, sh = shard0 + (int)blockIdx.y, tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int Ls = L / g;
    // the cache this kernel writes may still be read by the previous kernel (an attention pass)
    pdl_wait();
    pdl_trigger();

    const int pos = __ldg(positions + b);
    if (pos < 0 || pos >= max_pages * kPage) {
        if (tid == 0 && blockIdx.y == 0) atomicOr(status, kStatusIndex);
        return;
    }
    const int lp = pos / kPage;
    const int page = block_table ? __ldg(block_table + (size_t)b * max_pages + lp) : b * max_pages + lp;
    if (page < 0 || page >= num_pages) {   // recorded once, by the first CTA of the token
        if (tid == 0 && blockIdx.y == 0) atomicOr(status, kStatusIndex);
        return;
    }
    const int slot = pos % kPage;

    // butterfly span: the whole latent, or one shard's slice for the block-diagonal transform
    // (butterflies of stride h < L/g only pair indices of the same L/g-aligned block)
    const bool hadamard = transform == TPLA_TRANSFORM_HADAMARD || transform == TPLA_TRANSFORM_BLOCK_HADAMARD;
    const int hn = transform == TPLA_TRANSFORM_BLOCK_HADAMARD ? Ls : L;
    float xv = 0.f;                                   // x[tid] when L <= kThreads
    if (L <= kThreads) {
        if (tid < L) xv = __bfloat162float(latent_raw[(size_t)b * L + tid]);
        if (!hadamard && tid < L) x[tid] = xv;
    } else {
        for (int i = tid; i < L; i += kThreads) x[i] = __bfloat162float(latent_raw[(size_t)b * L + i]);
    }
    __syncthreads();

    if (hadamard && L <= kThreads) {
        // Radix-2 butterflies over hn = 2^k points (Sylvester order), one point per thread: the
        // pair (i, i + h) of stage h becomes (a + c, a - c).  Strides below 32 pair lanes of one
        // warp (shuffles); wider strides go through shared memory, alternating two buffers so
        // that one barrier per stage suffices.  Whole warps are idle when tid >= L (L >= 64).
        float v = xv;
        if (tid < L) {
            for (int h = 1; h < 32 && h < hn; h <<= 1) {
                const float o = __shfl_xor_sync(0xffffffffu, v, h);
                v = (tid & h) ? o - v : v + o;
            }
        }
        int buf = 0;
        for (int h = 32; h < hn; h <<= 1) {
            float* yb = buf ? y : x;
            if (tid < L) yb[tid] = v;
            __syncthreads();
            if (tid < L) {
                const float o = yb[tid ^ h];
                v = (tid & h) ? o - v : v + o;
            }
            buf ^= 1;
        }
        __syncthreads();   // every read of the last stage's buffer is done before y is written
        if (tid < L) y[tid] = v * (1.0f / sqrtf((float)hn));
    } else if (hadamard) {
        // in-place radix-2 butterflies of stride < hn (Sylvester order), then 1/sqrt(hn)
        for (int i = tid; i < L; i += kThreads) y[i] = x[i];
        __syncthreads();
        for (int hlen = 1; hlen < hn; hlen <<= 1) {
            for (int k = tid; k < L / 2; k += kThreads) {
                int i = (k / hlen) * 2 * hlen + (k % hlen);
                float a = y[i], c = y[i + hlen];
                y[i] = a + c;
                y[i + hlen] = a - c;
            }
            __syncthreads();
        }
        const float sc = 1.0f / sqrtf((float)hn);
        for (int i = tid; i < L; i += kThreads) y[i] *= sc;
    } else if (transform == TPLA_TRANSFORM_DENSE) {
        // y_i = sum_j R[i][j] x_j for the shard's rows: each warp takes four rows at a time,
        // coalesced over j, with the loads of kDenseBatch columns per row issued together
        constexpr int kDenseBatch = 16;
        for (int i0 = sh * Ls + warp * 4; i0 < (sh + 1) * Ls; i0 += (kThreads / 32) * 4) {
            const int nr = min(4, (sh + 1) * Ls - i0);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int j0 = 0; j0 < L; j0 += 32 * kDenseBatch) {
                float rv[4][kDenseBatch];
#pragma unroll
                for (int u = 0; u < kDenseBatch; ++u) {
                    const int j = j0 + u * 32 + lane;
#pragma unroll
                    for (int r = 0; r < 4; ++r)
                        rv[r][u] = (r < nr && j < L) ? __ldg(R_dense + (size_t)(i0 + r) * L + j) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < kDenseBatch; ++u) {
                    const int j = j0 + u * 32 + lane;
                    const float xj = j < L ? x[j] : 0.f;
#pragma unroll
                    for (int r = 0; r < 4; ++r) acc[r] = fmaf(rv[r][u], xj, acc[r]);
                }
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                for (int o = 16; o > 0; o >>= 1) acc[r] += __shfl_xor_sync(0xffffffffu, acc[r], o);
                if (lane == 0 && r < nr) y[i0 + r] = acc[r];
            }
        }
    } else {
        for (int i = tid; i < L; i += kThreads) y[i] = x[i];
    }
    __syncthreads();

    // sum of squares of this shard's slice: per 32-element chunk, then over the chunks
    const int y0 = sh * Ls;
    for (int c = warp; c < Ls / 32; c += kThreads / 32) {
        float v = y[y0 + c * 32 + lane];
        float ss = v * v;
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) part[c] = ss;
    }
    __syncthreads();
    if (tid == 0) {
        float ss = 0.f;
        for (int c = 0; c < Ls / 32; ++c) ss += part[c];
        inv_rms[0] = 1.0f / sqrtf(ss / (float)Ls + eps);
    }
    __syncthreads();

    for (int j = tid; j < Ls; j += kThreads) {
        float v = y[y0 + j] * inv_rms[0];
        if (norm_weight) v *= __ldg(norm_weight + y0 + j);
        ckv[(((size_t)page * g_out + blockIdx.y) * kPage + slot) * Ls + j] = __float2bfloat16_rn(v);
    }
    if (blockIdx.y == 0)
        for (int r = tid; r < R; r += kThreads)
            kpe[((size_t)page * kPage + slot) * R + r] = kpe_new[(size_t)b * R + r];
}

}  // namespace

cudaError_t launch_append(const tpla_dims_t& d, int shard, const __nv_bfloat16* latent_raw,
                          const __nv_bfloat16* kpe_new, int transform, const float* R_dense,
                          const float* norm_weight, float eps, const int32_t* positions,
                          const int32_t* block_table, __nv_bfloat16* ckv, __nv_bfloat16* kpe,
                          unsigned* status, cudaStream_t stream) {
    if (d.B == 0) return cudaSuccess;
    if (d.L > kMaxL) return cudaErrorNotSupported;
    const int shard0 = shard < 0 ? 0 : shard, gc = shard < 0 ? d.g : 1;
    return launch_pdl(append_kernel, dim3(d.B, gc), dim3(kThreads), 0, stream, d.L, d.R, d.g, shard0, gc,
                      d.max_pages_per_seq, d.num_pages, latent_raw, kpe_new, transform, R_dense, norm_weight, eps,
                      positions, block_table, ckv, kpe, status);
}

}  // namespace tpla
