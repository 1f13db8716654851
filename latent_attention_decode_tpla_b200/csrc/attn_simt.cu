// CUDA-core split-KV attention over the shard-contiguous latent cache.
//
// Per shard s of sequence b and head h (TPLA paper, Abstract: attention runs
// independently on each latent shard; edgentiq blog, "How TPLA Works":
// softmax slicing):
//     z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t)
//     o_{h,s} = sum_t softmax(z)_t c_{t,s}
// computed as an online (streaming) softmax over 64-token tiles, one split-KV
// segment at a time (schedule in tpla_internal.cuh).  This kernel uses plain
// fp32 FMAs on register tiles; it serves every supported shape (it is the
// path for g = 1, whose O does not fit in tensor memory beside S and the
// query) and is the yardstick the tcgen05 kernel is tested against.  One
// CTA = one worker x a group of 16 heads; every CTA of a worker walks the
// same units.
#include "tpla_internal.cuh"

#include <cuda_bf16.h>

namespace tpla {
namespace {

constexpr int kThreads = 256;
constexpr int kHG = 16;   // heads per CTA

// Register tiles.  QK^T: a warp takes one pair of heads, each lane two tokens (lane, lane + 32), so
// a thread holds a 2 x 2 block of scores and reads 4 elements of each query row (a broadcast) and
// of each cache row per 8-byte load; the query stays bf16 in shared memory (two CTAs fit an SM at
// L/g = 512) and the scale is applied to the finished dot products.  PV: a thread holds kHpt heads x kCpt latent columns and reads,
// per token, its heads' probabilities in one broadcast load and its columns of the cache row.
template <int LS, int RD>
struct SimtCfg {
    static constexpr int K = LS + RD;
    static constexpr int kRow = K + 4;               // bf16 per cached row: 8-byte aligned rows whose
                                                     // 64-bit loads from 16 consecutive rows hit distinct banks
    static constexpr int kCpt = LS >= 64 ? LS / 64 : 1;   // PV columns per thread
    static constexpr int kNcg = LS / kCpt;                // column groups
    static constexpr int kNhg = kThreads / kNcg;          // head groups
    static constexpr int kHpt = kHG / kNhg;               // PV heads per thread
    static constexpr int kProw = kHG + 4;                 // floats per token row of P (16-byte aligned)
    static_assert(K % 4 == 0 && kThreads % kNcg == 0 && kHG % kNhg == 0 && kHpt % 2 == 0, "thread map");
    static_assert(kThreads / 32 * 2 == kHG && kPage == 64, "QK^T map: one head pair per warp, two tokens per lane");
};

template <int LS, int RD>
struct SimtSmem {
    using C = SimtCfg<LS, RD>;
    __nv_bfloat16 q[kHG][C::kRow];                     // query rows [q~ slice | q_pe]
    __nv_bfloat16 c[kPage][C::kRow];                   // [c_s | k_pe] per token
    float p[kPage][C::kProw];                          // scores, then probabilities, token-major
    float alpha[kHG];
    float m[kHG];
    float l[kHG];
};

// n consecutive bf16 (n = 1, 2 or a multiple of 4; 8-byte aligned when n >= 4) from shared memory
template <int N>
__device__ __forceinline__ void ld_bf16(const __nv_bfloat16* src, float (&v)[N]) {
    if constexpr (N == 1) {
        v[0] = __bfloat162float(*src);
    } else if constexpr (N == 2) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(src));
        v[0] = f.x; v[1] = f.y;
    } else {
#pragma unroll
        for (int i = 0; i < N / 4; ++i) {
            const uint2 w = *reinterpret_cast<const uint2*>(src + 4 * i);
            const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.x));
            const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w.y));
            v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = b.x; v[4 * i + 3] = b.y;
        }
    }
}

template <int LS, int RD>
__global__ void __launch_bounds__(kThreads)
attn_simt_kernel(Plan p, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_pe,
                 const __nv_bfloat16* __restrict__ ckv, const __nv_bfloat16* __restrict__ kpe,
                 const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens,
                 Workspace ws) {
    using C = SimtCfg<LS, RD>;
    constexpr int K = C::K;
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& sm = *reinterpret_cast<SimtSmem<LS, RD>*>(smem_raw);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int w = blockIdx.x;
    const int h0 = blockIdx.y * kHG;
    // PV thread map
    const int cg = tid % C::kNcg, hg = tid / C::kNcg;
    const int j0 = cg * C::kCpt, hb = hg * C::kHpt;
    // the cache may have just been written by an append pass; the next kernel launches when the
    // CTAs of this one have exited (no early trigger)
    pdl_wait();

    const long long V = warp_total_weight(seq_lens, p);
    if (V == 0) return;
    const long long lo = warp_unit_at_weight(seq_lens, p, unit_lo(w, V, p.W));
    const long long hi = warp_unit_at_weight(seq_lens, p, unit_lo(w + 1, V, p.W));
    if (lo >= hi) {
        // a worker with no units leaves a zero-weight partial in its slot: the merge may count it
        // as a segment of the pair it falls inside
        for (int i = threadIdx.x; i < kHG && h0 + i < p.H; i += blockDim.x) ws.part_lse[(size_t)w * p.H + h0 + i] = -INFINITY;
        return;
    }
    UnitPos pos = warp_locate_unit(seq_lens, p.B, p.max_pages, p.gc, lo);

    float acc[C::kHpt][C::kCpt];
    for (long long u = lo; u < hi; ++u) {
        const bool seg_begin = (u == lo) || pos.tile == 0;
        const bool seg_end = (u == hi - 1) || pos.tile == pos.ntiles - 1;
        const int shard = p.shard0 + pos.s;
        if (seg_begin) {
            __syncthreads();
            (void)effective_len(seq_lens, pos.b, p.max_pages, p.status);   // records a clamp
            for (int i = tid; i < kHG * K; i += kThreads) {
                int h = i / K, k = i % K, hgl = h0 + h;
                __nv_bfloat16 v = __float2bfloat16_rn(0.f);
                if (hgl < p.H) {
                    v = k < LS ? q[((size_t)pos.b * p.H + hgl) * p.L + (size_t)shard * LS + k]
                               : q_pe[((size_t)pos.b * p.H + hgl) * RD + (k - LS)];
                }
                sm.q[h][k] = v;
            }
            if (tid < kHG) { sm.m[tid] = -INFINITY; sm.l[tid] = 0.f; }
#pragma unroll
            for (int a = 0; a < C::kHpt; ++a)
#pragma unroll
                for (int b = 0; b < C::kCpt; ++b) acc[a][b] = 0.f;
        }
        const int valid = min(kPage, pos.T - pos.tile * kPage);
        const int page = page_lookup(block_table, pos.b, pos.tile, p.max_pages, p.num_pages, p.status);
        __syncthreads();
        // stage the tile in 8-byte pieces: latent slice of this shard, then the shared RoPE key;
        // rows past the sequence end (or of a missing page) are zero
        {
            const uint2* src_c = reinterpret_cast<const uint2*>(
                ckv + (((size_t)(page < 0 ? 0 : page) * p.g + shard) * kPage) * LS);
            const uint2* src_k = reinterpret_cast<const uint2*>(kpe + (size_t)(page < 0 ? 0 : page) * kPage * RD);
            constexpr int WC = LS / 4, WK = RD / 4;
            for (int i = tid; i < kPage * (WC + WK); i += kThreads) {
                int t = i / (WC + WK), k = i % (WC + WK);
                uint2 v = make_uint2(0u, 0u);
                if (t < valid && page >= 0) v = k < WC ? __ldg(src_c + t * WC + k) : __ldg(src_k + t * WK + (k - WC));
                reinterpret_cast<uint2*>(&sm.c[t][0])[k] = v;
            }
        }
        __syncthreads();
        // scores (log2 domain): s = (scale*log2e) * (q . [c | k_pe]) for heads 2*warp, 2*warp + 1 and
        // tokens lane, lane + 32; even and odd k in separate sums for more independent FMAs
        {
            const int ha = 2 * warp;
            const __nv_bfloat16* qa = &sm.q[ha][0];
            const __nv_bfloat16* qb = &sm.q[ha + 1][0];
            const __nv_bfloat16* r0 = &sm.c[lane][0];
            const __nv_bfloat16* r1 = &sm.c[lane + 32][0];
            float s[2][2][2] = {};   // [head][token][parity]
#pragma unroll 4
            for (int k4 = 0; k4 < K / 4; ++k4) {
                float av[4], bv[4];
                ld_bf16<4>(qa + 4 * k4, av);
                ld_bf16<4>(qb + 4 * k4, bv);
                const float4 a = make_float4(av[0], av[1], av[2], av[3]), b = make_float4(bv[0], bv[1], bv[2], bv[3]);
                float c0[4], c1[4];
                ld_bf16<4>(r0 + 4 * k4, c0);
                ld_bf16<4>(r1 + 4 * k4, c1);
                s[0][0][0] = fmaf(a.x, c0[0], s[0][0][0]); s[0][0][1] = fmaf(a.y, c0[1], s[0][0][1]);
                s[0][0][0] = fmaf(a.z, c0[2], s[0][0][0]); s[0][0][1] = fmaf(a.w, c0[3], s[0][0][1]);
                s[0][1][0] = fmaf(a.x, c1[0], s[0][1][0]); s[0][1][1] = fmaf(a.y, c1[1], s[0][1][1]);
                s[0][1][0] = fmaf(a.z, c1[2], s[0][1][0]); s[0][1][1] = fmaf(a.w, c1[3], s[0][1][1]);
                s[1][0][0] = fmaf(b.x, c0[0], s[1][0][0]); s[1][0][1] = fmaf(b.y, c0[1], s[1][0][1]);
                s[1][0][0] = fmaf(b.z, c0[2], s[1][0][0]); s[1][0][1] = fmaf(b.w, c0[3], s[1][0][1]);
                s[1][1][0] = fmaf(b.x, c1[0], s[1][1][0]); s[1][1][1] = fmaf(b.y, c1[1], s[1][1][1]);
                s[1][1][0] = fmaf(b.z, c1[2], s[1][1][0]); s[1][1][1] = fmaf(b.w, c1[3], s[1][1][1]);
            }
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                for (int tt = 0; tt < 2; ++tt) {
                    const int t = lane + 32 * tt;
                    sm.p[t][ha + hh] = t < valid ? (s[hh][tt][0] + s[hh][tt][1]) * p.scale_log2 : -INFINITY;
                }
        }
        __syncthreads();
        // online softmax, one warp per head
        for (int h = warp; h < kHG; h += kThreads / 32) {
            float s0 = sm.p[lane][h], s1 = sm.p[lane + 32][h];
            float mt = fmaxf(s0, s1);
            for (int o = 16; o > 0; o >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, o));
            float m_old = sm.m[h];
            float m_new = fmaxf(m_old, mt);
            float e0 = exp2f(s0 - m_new), e1 = exp2f(s1 - m_new);
            float ls = e0 + e1;
            for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
            sm.p[lane][h] = e0;
            sm.p[lane + 32][h] = e1;
            if (lane == 0) {
                float alpha = exp2f(m_old - m_new);
                sm.alpha[h] = alpha;
                sm.l[h] = sm.l[h] * alpha + ls;
                sm.m[h] = m_new;
            }
        }
        __syncthreads();
        // o = alpha * o + P C over this thread's heads and columns (rows past `valid` have p = 0
        // and zeroed cache rows)
#pragma unroll
        for (int a = 0; a < C::kHpt; ++a) {
            const float al = sm.alpha[hb + a];
#pragma unroll
            for (int b = 0; b < C::kCpt; ++b) acc[a][b] *= al;
        }
#pragma unroll 2
        for (int t = 0; t < kPage; ++t) {
            float pv[C::kHpt], cv[C::kCpt];
#pragma unroll
            for (int a = 0; a < C::kHpt; a += 2) {
                const float2 pp = *reinterpret_cast<const float2*>(&sm.p[t][hb + a]);
                pv[a] = pp.x; pv[a + 1] = pp.y;
            }
            ld_bf16<C::kCpt>(&sm.c[t][j0], cv);
#pragma unroll
            for (int a = 0; a < C::kHpt; ++a)
#pragma unroll
                for (int b = 0; b < C::kCpt; ++b) acc[a][b] = fmaf(pv[a], cv[b], acc[a][b]);
        }
        if (seg_end) {
            // the segment started at max(lo, unit of tile 0 of this (b, s))
            const int sl = u - pos.tile >= lo ? p.W + pos.b * p.gc + pos.s : w;
            __syncthreads();
#pragma unroll
            for (int a = 0; a < C::kHpt; ++a) {
                const int h = hb + a;
                if (h0 + h < p.H) {
                    const float inv = 1.0f / sm.l[h];
                    float* dst = ws.part_o + ((size_t)sl * p.H + h0 + h) * LS + j0;
#pragma unroll
                    for (int b = 0; b < C::kCpt; ++b) dst[b] = acc[a][b] * inv;
                }
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
