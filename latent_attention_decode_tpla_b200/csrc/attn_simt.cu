// CUDA-core split-KV attention over the shard-contiguous latent cache.
//
// Per shard s of sequence b and head h (TPLA paper, Abstract: attention runs
// independently on each latent shard; edgentiq blog, "How TPLA Works":
// softmax slicing):
//     z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t)
//     o_{h,s} = sum_t softmax(z)_t c_{t,s}
// computed as an online (streaming) softmax over 64-token tiles, one split-KV
// segment at a time (schedule in tpla_internal.cuh).  This kernel uses plain
// fp32 FMAs; it serves every supported shape and is the yardstick the
// tcgen05 kernel is tested against.  One CTA = one worker x a group of 16
// heads; every CTA of a worker walks the same units.
#include "tpla_internal.cuh"

#include <cuda_bf16.h>

namespace tpla {
namespace {

constexpr int kThreads = 256;
constexpr int kHG = 16;   // heads per CTA

template <int LS, int RD>
struct SimtSmem {
    static constexpr int kRow = LS + RD + 2;          // bf16 per cached row (+2: odd word stride)
    float q[kHG][LS + RD];                             // scaled query rows
    __nv_bfloat16 c[kPage][kRow];                      // [c_s | k_pe] per token
    float p[kHG][kPage];                               // scores, then probabilities
    float alpha[kHG];
    float m[kHG];
    float l[kHG];
};

template <int LS, int RD>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(Plan p, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_pe,
                 const __nv_bfloat16* __restrict__ ckv, const __nv_bfloat16* __restrict__ kpe,
                 const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens,
                 Workspace ws) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SimtSmem<LS, RD>*>(smem_raw);
    constexpr int K = LS + RD;
    constexpr int NACC = kHG * LS / kThreads > 0 ? kHG * LS / kThreads : 1;
    static_assert(kHG * LS % kThreads == 0 || kHG * LS < kThreads, "thread map");

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int w = blockIdx.x;
    const int h0 = blockIdx.y * kHG;
    // the cache may have just been written by an append pass; the next kernel launches when the
    // CTAs of this one have exited (no early trigger)
    pdl_wait();

    const long long U = warp_total_units(seq_lens, p.B, p.max_pages, p.gc);
    if (U == 0) return;
    const long long lo = unit_lo(w, U, p.W), hi = unit_lo(w + 1, U, p.W);
    if (lo >= hi) {
        // a worker with no units leaves a zero-weight partial in its slot: the merge may count it
        // as a segment of the pair it falls inside
        for (int i = threadIdx.x; i < kHG && h0 + i < p.H; i += blockDim.x) ws.part_lse[(size_t)w * p.H + h0 + i] = -INFINITY;
        return;
    }
    UnitPos pos = warp_locate_unit(seq_lens, p.B, p.max_pages, p.gc, lo);

    float acc[NACC];
    for (long long u = lo; u < hi; ++u) {
        const bool seg_begin = (u == lo) || pos.tile == 0;
        const bool seg_end = (u == hi - 1) || pos.tile == pos.ntiles - 1;
        const int shard = p.shard0 + pos.s;
        if (seg_begin) {
            __syncthreads();
            (void)effective_len(seq_lens, pos.b, p.max_pages, p.status);   // records a clamp
            for (int i = tid; i < kHG * K; i += kThreads) {
                int h = i / K, k = i % K, hg = h0 + h;
                float v = 0.f;
                if (hg < p.H) {
                    v = k < LS ? __bfloat162float(q[((size_t)pos.b * p.H + hg) * p.L + (size_t)shard * LS + k])
                               : __bfloat162float(q_pe[((size_t)pos.b * p.H + hg) * RD + (k - LS)]);
                }
                sm.q[h][k] = v * p.scale_log2;
            }
            if (tid < kHG) { sm.m[tid] = -INFINITY; sm.l[tid] = 0.f; }
#pragma unroll
            for (int a = 0; a < NACC; ++a) acc[a] = 0.f;
        }
        const int valid = min(kPage, pos.T - pos.tile * kPage);
        const int page = page_lookup(block_table, pos.b, pos.tile, p.max_pages, p.num_pages, p.status);
        __syncthreads();
        // stage the tile: latent slice of this shard, then the shared RoPE key
        {
            const uint32_t* src_c = reinterpret_cast<const uint32_t*>(
                ckv + (((size_t)(page < 0 ? 0 : page) * p.g + shard) * kPage) * LS);
            const uint32_t* src_k = reinterpret_cast<const uint32_t*>(kpe + (size_t)(page < 0 ? 0 : page) * kPage * RD);
            constexpr int WC = LS / 2, WK = RD / 2;
            for (int i = tid; i < kPage * (WC + WK); i += kThreads) {
                int t = i / (WC + WK), k = i % (WC + WK);
                uint32_t v = 0;
                if (t < valid && page >= 0) v = k < WC ? __ldg(src_c + t * WC + k) : __ldg(src_k + t * WK + (k - WC));
                reinterpret_cast<uint32_t*>(&sm.c[t][0])[k] = v;
            }
        }
        __syncthreads();
        // scores (log2 domain): s = (scale*log2e) * (q . [c | k_pe]); each thread takes the
        // kSc (head, token) pairs tid + kThreads * i with the same token t, interleaved
        {
            constexpr int kSc = kHG * kPage / kThreads;       // 4
            static_assert(kHG * kPage % kThreads == 0 && kThreads % kPage == 0, "score map");
            const int t = tid % kPage, hb = tid / kPage;      // heads hb + (kThreads / kPage) * i
            const __nv_bfloat162* row = reinterpret_cast<const __nv_bfloat162*>(&sm.c[t][0]);
            float d0[kSc], d1[kSc];
#pragma unroll
            for (int i = 0; i < kSc; ++i) d0[i] = d1[i] = 0.f;
#pragma unroll 4
            for (int k = 0; k < K / 2; ++k) {
                const float2 cv = __bfloat1622float2(row[k]);
#pragma unroll
                for (int i = 0; i < kSc; ++i) {
                    const int h = hb + (kThreads / kPage) * i;
                    d0[i] = fmaf(sm.q[h][2 * k], cv.x, d0[i]);
                    d1[i] = fmaf(sm.q[h][2 * k + 1], cv.y, d1[i]);
                }
            }
#pragma unroll
            for (int i = 0; i < kSc; ++i)
                sm.p[hb + (kThreads / kPage) * i][t] = t < valid ? d0[i] + d1[i] : -INFINITY;
        }
        __syncthreads();
        // online softmax, one warp per head
        for (int h = warp; h < kHG; h += kThreads / 32) {
            float s0 = sm.p[h][lane], s1 = sm.p[h][lane + 32];
            float mt = fmaxf(s0, s1);
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            float m_old = sm.m[h];
            float m_new = fmaxf(m_old, mt);
            float e0 = exp2f(s0 - m_new), e1 = exp2f(s1 - m_new);
            float ls = e0 + e1;
            for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            sm.p[h][lane] = e0;
            sm.p[h][lane + 32] = e1;
            if (lane == 0) {
                float alpha = exp2f(m_old - m_new);
                sm.alpha[h] = alpha;
                sm.l[h] = sm.l[h] * alpha + ls;
                sm.m[h] = m_new;
            }
        }
        __syncthreads();
        // o = alpha * o + P C, with the token loop outside so that the NACC accumulators give
        // independent FMAs (rows past `valid` have p = 0 and zeroed cache rows)
#pragma unroll
        for (int a = 0; a < NACC; ++a) {
            const int flat = tid + kThreads * a;
            const int h = flat / LS;
            if (h < kHG) acc[a] *= sm.alpha[h];
        }
        for (int t = 0; t < kPage; ++t) {
#pragma unroll
            for (int a = 0; a < NACC; ++a) {
                const int flat = tid + kThreads * a;
                const int h = flat / LS, j = flat % LS;
                if (h < kHG) acc[a] = fmaf(sm.p[h][t], __bfloat162float(sm.c[t][j]), acc[a]);
            }
        }
        if (seg_end) {
            // the segment started at max(lo, unit of tile 0 of this (b, s))
            const long long seg_first = u - pos.tile < lo ? lo : u - pos.tile;
            const int sl = (seg_first == lo) ? w : p.W + pos.b * p.gc + pos.s;
            __syncthreads();
#pragma unroll
            for (int a = 0; a < NACC; ++a) {
                int flat = tid + kThreads * a;
                int h = flat / LS, j = flat % LS;
                if (h < kHG && h0 + h < p.H)
                    ws.part_o[((size_t)sl * p.H + h0 + h) * LS + j] = acc[a] / sm.l[h];
            }
            if (tid < kHG && h0 + tid < p.H)
                ws.part_lse[(size_t)sl * p.H + h0 + tid] = sm.m[tid] + log2f(sm.l[tid]);
        }
        advance_unit(pos, seq_lens, p.B, p.max_pages, p.gc);
    }
}

template <int LS, int RD>
cudaError_t launch_t(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                     const __nv_bfloat16* ckv, const __nv_bfloat16* kpe, const int32_t* bt,
                     const int32_t* seq_lens, Workspace ws, cudaStream_t stream) {
    const size_t smem = sizeof(SimtSmem<LS, RD>);
    auto kern = attn_simt_kernel<LS, RD>;
    static unsigned long long attr_done = 0;
    cudaError_t e = set_smem_once(kern, smem, &attr_done);
    if (e != cudaSuccess) return e;
    dim3 grid(p.W, (p.H + kHG - 1) / kHG);
    return launch_pdl(kern, grid, dim3(kThreads), smem, stream, p, q, q_pe, ckv, kpe, bt, seq_lens, ws);
}

template <int LS>
cudaError_t launch_r(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                     const __nv_bfloat16* ckv, const __nv_bfloat16* kpe, const int32_t* bt,
                     const int32_t* seq_lens, Workspace ws, cudaStream_t stream) {
    switch (p.R) {
        case 16: return launch_t<LS, 16>(p, q, q_pe, ckv, kpe, bt, seq_lens, ws, stream);
        case 32: return launch_t<LS, 32>(p, q, q_pe, ckv, kpe, bt, seq_lens, ws, stream);
        case 64: return launch_t<LS, 64>(p, q, q_pe, ckv, kpe, bt, seq_lens, ws, stream);
    }
    return cudaErrorNotSupported;
}

}  // namespace

cudaError_t launch_attention_simt(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                  const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                  const int32_t* block_table, const int32_t* seq_lens,
                                  Workspace ws, cudaStream_t stream) {
    switch (p.Ls) {
        case 32: return launch_r<32>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, stream);
        case 64: return launch_r<64>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, stream);
        case 128: return launch_r<128>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, stream);
        case 256: return launch_r<256>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, stream);
        case 512: return launch_r<512>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, stream);
    }
    return cudaErrorNotSupported;
}

}  // namespace tpla
