// Combine: split-KV merge, W_UV up-projection, and the sum over shards, in one kernel.
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
// One CTA per (head h, dv slice, group of Bc sequences):
//   1. one thread starts the bulk copy of the CTA's W_UV rows into shared
//      memory (a single copy when the slice is the whole dv);
//   2. one warp finds, for each (sequence, shard) pair of the group, the
//      workers holding its first and last tile (a prefix sum over seq_lens);
//   3. every thread (or group of up to 8 lanes, when there are few pairs)
//      merges one 4-float piece of one pair's row over that pair's segments
//      in a single pass (running maximum and rescale), so all partial and
//      log-sum-exp loads are independent;
//   4. the projection keeps kRows rows x 8 columns per lane in registers (one
//      16-byte W_UV load per row of the reduction for 64 FMAs), sums the lanes'
//      parts by shuffles and the warps' parts through shared memory.
// The partials were just written by the attention kernel and come from L2.
#include "tpla_internal.cuh"
#include "sm100_ptx.cuh"

namespace tpla {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr size_t kWSmemBudget = 160 * 1024;    // bytes of W_UV staged per CTA (a whole head of 512 x 128 fits)
constexpr int kMergeTarget = 2048;             // merged floats per CTA the group size aims at
constexpr int kMaxRows = 8;                    // merged rows projected together, at most
constexpr int kMaxPairs = 64;                  // (sequence, shard) pairs per CTA
constexpr int kBatch = 16;                     // segments whose loads a thread issues together

// The owner of the unit whose weighted start is v (the largest w with floor(w V / W) <= v), in
// 32-bit arithmetic when (W + 1) V fits (64-bit integer division is emulated and slow), else in 64
// bits.
struct UnitMath {
    long long V;
    int W;
    bool small;
    __device__ int worker(long long v) const {
        return small ? (int)(((unsigned)(v + 1) * (unsigned)W - 1u) / (unsigned)V) : unit_worker(v, V, W);
    }
};

struct PairInfo {
    int wf, wl;        // workers holding the pair's first and last tile (wl < wf: empty sequence)
    int first_slot;    // slot of the first segment (the one that starts at tile 0)
};

template <int kRows>
__global__ void __launch_bounds__(kThreads)
combine_kernel(Plan p, int Bc, int dsub, const int32_t* __restrict__ seq_lens, Workspace ws,
               const __nv_bfloat16* __restrict__ w_uv, float* __restrict__ out, uint64_t wait_cycles) {
    extern __shared__ __align__(128) uint8_t csm[];
    __shared__ PairInfo pinfo[kMaxPairs];
    __shared__ __align__(8) uint64_t wbar;
    const int Lc = p.gc * p.Ls;
    const int h = blockIdx.x, d0 = blockIdx.y * dsub, b0 = blockIdx.z * Bc;
    const int nb = min(Bc, p.B - b0);
    const int npairs = nb * p.gc;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const bool project = w_uv != nullptr;
    // shared memory: W_UV rows [Lc][dsub] bf16 | merged rows [Bc][Lc] fp32 | warps' partial sums
    // [kWarps][kRows][dsub] fp32
    __nv_bfloat16* w_s = reinterpret_cast<__nv_bfloat16*>(csm);
    const size_t w_bytes = project ? (size_t)Lc * dsub * 2 : 0;
    float* o_s = reinterpret_cast<float*>(csm + w_bytes);
    float* red = o_s + (size_t)Bc * Lc;

    // 1. W_UV[h][shard0*Ls + j][d0 .. d0+dsub) for j < Lc
    if (project && warp == 0) {
        if (lane == 0) {
            mbar_init(smem_addr(&wbar), 1);
            fence_barrier_init();
            mbar_arrive_expect_tx(smem_addr(&wbar), (uint32_t)w_bytes);
        }
        __syncwarp();
        const __nv_bfloat16* src = w_uv + ((size_t)h * p.L + (size_t)p.shard0 * p.Ls) * p.dv + d0;
        if (dsub == p.dv) {
            if (lane == 0) bulk_load(smem_addr(w_s), src, (uint32_t)w_bytes, smem_addr(&wbar));
        } else {
            for (int j = lane; j < Lc; j += 32)
                bulk_load(smem_addr(w_s + (size_t)j * dsub), src + (size_t)j * p.dv, (uint32_t)(dsub * 2),
                          smem_addr(&wbar));
        }
    }
    // 2. first and last worker of each pair: prefix sum of the unit weights over the sequences
    // before b (the schedule in tpla_internal.cuh)
    if (warp == (project ? 1 : 0)) {
        UnitMath um;
        um.V = warp_total_weight(seq_lens, p);
        um.W = p.W;
        um.small = um.V < (1ll << 32) / (p.W + 1);
        long long before = 0;                         // weight of sequences < base
        for (int base = 0; base < b0 + nb; base += 32) {
            const int b = base + lane;
            int nt = 0, c = 1;
            if (b < b0 + nb) {
                int T = __ldg(seq_lens + b);
                T = T < 0 ? 0 : (T > p.max_pages * kPage ? p.max_pages * kPage : T);
                nt = tiles_of_len(T);
                c = unit_weight(p, T);
            }
            long long incl = (long long)nt * p.gc * c;   // inclusive scan over the lanes
            for (int o = 1; o < 32; o <<= 1) {
                const long long v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b >= b0 && b < b0 + nb) {
                const long long vb = before + incl - (long long)nt * p.gc * c;   // weighted start of b
                for (int s = 0; s < p.gc; ++s) {
                    PairInfo pi;
                    if (nt == 0) {
                        pi.wf = 0; pi.wl = -1; pi.first_slot = 0;
                    } else {
                        const long long v0 = vb + (long long)s * nt * c;
                        pi.wf = um.worker(v0);
                        pi.wl = um.worker(v0 + (long long)(nt - 1) * c);
                        pi.first_slot = p.W + b * p.gc + s;
                    }
                    pinfo[(b - b0) * p.gc + s] = pi;
                }
            }
            before += __shfl_sync(0xffffffffu, incl, 31);
        }
    }
    __syncthreads();
    // the partials come from the previous grid (the attention pass of this call): wait for it, then
    // let the next kernel launch
    pdl_wait();
    pdl_trigger();

    // 3. merge: one float4 of one pair's row per group of nsplit adjacent lanes; the lanes of a
    // group take every nsplit-th segment and combine their partial merges by shuffles (when there
    // are fewer items than threads, e.g. one long sequence split over many workers)
    const int q4 = p.Ls / 4;
    const int items = npairs * q4;
    int nsplit = 1;
    while (nsplit < 8 && items * nsplit * 2 <= kThreads) nsplit *= 2;
    const int t = tid % nsplit;
    for (int base = 0; base < items; base += kThreads / nsplit) {   // same trip count in every lane
        const int i = base + tid / nsplit;
        const bool active = i < items;
        const int pr = active ? i / q4 : 0, j = active ? (i % q4) * 4 : 0;
        const PairInfo pi = pinfo[pr];
        float M = -INFINITY, den = 0.f;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        // segments: the first one, then one per later worker up to the last.  A worker with an
        // empty range (possible when there are fewer units than workers) left lse = -inf in its
        // slot, so its weight is 0 and its partial, never written, is not read into the sum.  The
        // loads of a batch of kBatch segments are issued together, then folded in.
        const int kbeg = active ? pi.wf + t : 1, kend = active ? pi.wl : 0;
        for (int kb = kbeg; kb <= kend; kb += kBatch * nsplit) {
            float lse[kBatch];
            float4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int k = kb + u * nsplit;
                lse[u] = -INFINITY;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (k <= kend) {
                    const size_t slot = (size_t)(k == pi.wf ? pi.first_slot : k);
                    lse[u] = __ldg(ws.part_lse + slot * p.H + h);
                    v[u] = __ldg(reinterpret_cast<const float4*>(ws.part_o + (slot * p.H + h) * p.Ls + j));
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                if (lse[u] == -INFINITY) continue;
                const float Mn = fmaxf(M, lse[u]);
                const float a = exp2f(M - Mn), wk = exp2f(lse[u] - Mn);   // exp2f(-inf) = 0 on the first one
                den = den * a + wk;
                acc.x = acc.x * a + wk * v[u].x;
                acc.y = acc.y * a + wk * v[u].y;
                acc.z = acc.z * a + wk * v[u].z;
                acc.w = acc.w * a + wk * v[u].w;
                M = Mn;
            }
        }
        for (int off = 1; off < nsplit; off <<= 1) {   // combine the group's partial merges
            const float Mo = __shfl_xor_sync(0xffffffffu, M, off);
            const float dno = __shfl_xor_sync(0xffffffffu, den, off);
            const float4 ao = make_float4(__shfl_xor_sync(0xffffffffu, acc.x, off), __shfl_xor_sync(0xffffffffu, acc.y, off),
                                          __shfl_xor_sync(0xffffffffu, acc.z, off), __shfl_xor_sync(0xffffffffu, acc.w, off));
            const float Mn = fmaxf(M, Mo);
            const float e1 = M == -INFINITY ? 0.f : exp2f(M - Mn), e2 = Mo == -INFINITY ? 0.f : exp2f(Mo - Mn);
            den = den * e1 + dno * e2;
            acc.x = acc.x * e1 + ao.x * e2;
            acc.y = acc.y * e1 + ao.y * e2;
            acc.z = acc.z * e1 + ao.z * e2;
            acc.w = acc.w * e1 + ao.w * e2;
            M = Mn;
        }
        if (!active || t != 0) continue;
        const int bl = pr / p.gc, s = pr % p.gc;
        const float inv = pi.wl >= pi.wf ? 1.0f / den : 0.f;
        const float4 r = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (project) {
            *reinterpret_cast<float4*>(o_s + (size_t)bl * Lc + s * p.Ls + j) = r;
        } else {
            *reinterpret_cast<float4*>(out + ((size_t)(b0 + bl) * p.H + h) * Lc + s * p.Ls + j) = r;
        }
    }
    if (!project) return;
    for (int i = nb * Lc + tid; i < Bc * Lc; i += kThreads) o_s[i] = 0.f;   // rows past the batch
    {   // wait for W_UV (bounded; a time-out is recorded in the device status)
        const long long t0 = clock64();
        while (!mbar_try_wait(smem_addr(&wbar), 0)) {
            if ((uint64_t)(clock64() - t0) > wait_cycles) {
                if (tid == 0) atomicOr(p.status, kStatusTimeout);
                break;
            }
        }
    }
    __syncthreads();

    // 4. projection: out[b][d0 + 8c + e] = sum_j o[b][j] * W[j][8c + e].  Lane = (column group c of 8,
    // part of this warp's slice of j).
    const int cg = dsub / 8, ppw = 32 / cg;
    const int cgi = lane % cg, part = lane / cg;
    const int nparts = kWarps * ppw;
    const int jpp = (Lc + nparts - 1) / nparts;
    const int j0 = min(Lc, (warp * ppw + part) * jpp), j1 = min(Lc, j0 + jpp);
    for (int r0 = 0; r0 < nb; r0 += kRows) {
        float acc[kRows][8];
#pragma unroll
        for (int r = 0; r < kRows; ++r)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[r][e] = 0.f;
        const float* orow = o_s + (size_t)r0 * Lc;
#pragma unroll 2
        for (int j = j0; j < j1; ++j) {
            const uint4 wv = *reinterpret_cast<const uint4*>(w_s + (size_t)j * dsub + cgi * 8);
            const uint32_t wwords[4] = {wv.x, wv.y, wv.z, wv.w};
            float wf[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                wf[2 * e] = __uint_as_float(wwords[e] << 16);
                wf[2 * e + 1] = __uint_as_float(wwords[e] & 0xFFFF0000u);
            }
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                const float ov = orow[(size_t)r * Lc + j];   // rows past nb are zero
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[r][e] = fmaf(ov, wf[e], acc[r][e]);
            }
        }
        for (int off = cg; off < 32; off <<= 1)
#pragma unroll
            for (int r = 0; r < kRows; ++r)
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[r][e] += __shfl_xor_sync(0xffffffffu, acc[r][e], off);
        if (part == 0) {
#pragma unroll
            for (int r = 0; r < kRows; ++r) {
                float4* dst = reinterpret_cast<float4*>(red + ((size_t)warp * kRows + r) * dsub + cgi * 8);
                dst[0] = make_float4(acc[r][0], acc[r][1], acc[r][2], acc[r][3]);
                dst[1] = make_float4(acc[r][4], acc[r][5], acc[r][6], acc[r][7]);
            }
        }
        __syncthreads();
        for (int i = tid; i < kRows * dsub; i += kThreads) {
            const int r = i / dsub, dd = i % dsub;
            if (r0 + r < nb) {
                float sum = 0.f;
#pragma unroll
                for (int w = 0; w < kWarps; ++w) sum += red[((size_t)w * kRows + r) * dsub + dd];
                out[((size_t)(b0 + r0 + r) * p.H + h) * p.dv + d0 + dd] = sum;
            }
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_combine(const Plan& p, const int32_t* seq_lens, const __nv_bfloat16* w_uv,
                           float* out, Workspace ws, cudaStream_t stream) {
    if (p.B == 0) return cudaSuccess;
    const int Lc = p.gc * p.Ls;
    // sequences per CTA: about kMergeTarget merged floats per CTA; when projecting, a power of two
    // up to kMaxRows, or whole chunks of kMaxRows rows
    int Bc = kMergeTarget / Lc;
    Bc = Bc < 1 ? 1 : (Bc > p.B ? p.B : Bc);
    int rows = kMaxRows;
    if (w_uv) {
        rows = 1;
        while (rows < Bc && rows < kMaxRows) rows *= 2;
        Bc = (Bc + rows - 1) / rows * rows;
    }
    while (Bc * p.gc > kMaxPairs) Bc = Bc > rows ? Bc - rows : Bc / 2;
    if (Bc < 1) return cudaErrorNotSupported;
    // dv slice: the widest 8 * 2^k columns (at most 256) that divide dv and whose W_UV rows fit the
    // shared-memory budget (dv % 8 == 0)
    int dsub = 8;
    if (w_uv) {
        while (dsub * 2 <= 256 && p.dv % (dsub * 2) == 0 && (size_t)Lc * dsub * 4 <= kWSmemBudget) dsub *= 2;
        if ((size_t)Lc * dsub * 2 > kWSmemBudget) return cudaErrorNotSupported;
    }
    const size_t smem = (w_uv ? (size_t)Lc * dsub * 2 + (size_t)kWarps * rows * dsub * sizeof(float) : 0) +
                        (size_t)Bc * Lc * sizeof(float);
    constexpr size_t kMaxDyn = 200 * 1024;
    if (smem > kMaxDyn) return cudaErrorNotSupported;
    dim3 grid(p.H, w_uv ? p.dv / dsub : 1, (p.B + Bc - 1) / Bc);
    const uint64_t wait_cycles = 2ull * 1000 * 1000 * 1000;   // about a second at the SM clock
    auto launch = [&](auto kern, unsigned long long* done) -> cudaError_t {
        cudaError_t e = set_smem_once(kern, kMaxDyn, done);
        if (e != cudaSuccess) return e;
        return launch_pdl(kern, grid, dim3(kThreads), smem, stream, p, Bc, dsub, seq_lens, ws, w_uv, out, wait_cycles);
    };
    static unsigned long long done[4] = {0, 0, 0, 0};
    switch (rows) {
        case 1: return launch(combine_kernel<1>, &done[0]);
        case 2: return launch(combine_kernel<2>, &done[1]);
        case 4: return launch(combine_kernel<4>, &done[2]);
        default: return launch(combine_kernel<8>, &done[3]);
    }
}

}  // namespace tpla
