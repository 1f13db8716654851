// tcgen05 / TMEM / TMA split-KV attention over the shard-contiguous latent
// cache, for sm_100a (B200).
//
// What it computes (TPLA paper, Abstract; edgentiq blog "How TPLA Works"):
// for every shard s of sequence b and every head h
//     z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t)
//     o_{h,s} = sum_t softmax_t(z) c_{t,s}
// as an online softmax over 64-token tiles of one split-KV segment
// (schedule in tpla_internal.cuh); the result per segment is the normalised
// o and log2-sum-exp per head, merged later by the combine kernel.
//
// All heads of a sequence share every cache row, so both contractions are
// dense with the heads as the MMA M dimension (M = 128; fewer heads are
// padded):
//     S[h, t]  = Q[h, :] . [C_s | K_pe][t, :]^T     M=128, N=64,  K=Ls+R
//     O[h, :] += P[h, t] . C_s[t, :]                M=128, N=Ls,  K=64
// One 64-token tile is TMA-loaded once into 128B-swizzled shared memory and
// is the K-major B operand of the first MMA and the MN-major B operand of
// the second.  Q and P are the A operands and live in tensor memory, so the
// shared-memory bandwidth goes to the cache stream only.  O (fp32) and S
// (fp32) accumulate in tensor memory.
//
// Precision: QK^T multiplies the bf16 inputs as they are.  For PV the
// probabilities are rounded to fp16 (11 significant bits) rather than bf16
// (8 bits): rounding P to bf16 alone costs about 1.2e-3 relative RMS error on
// outputs of short sequences, fp16 about 1.5e-4.  One MMA never mixes the
// two types, so after QK^T of a tile has completed, the softmax warps convert
// that tile's latent rows in shared memory from bf16 to fp16 in place (each
// bf16 value of the RMS-normalised cache is exactly an fp16 value unless its
// magnitude is below 2^-14), zero the rows past the end of the sequence, and
// only then release the tile to PV.
//
// Warp roles (192 threads): warp 0 issues TMA loads into a ring of NST
// stages; warp 1 allocates tensor memory and issues the MMAs (one thread);
// warps 2-5 own the 128 TMEM lanes (one head row per thread) and do the
// softmax, the O rescale, the P store and the epilogue.  The MMA warp issues
// QK^T of tile j before PV of tile j-1 so the tensor pipe works while the
// softmax warps exponentiate.  O is rescaled only when a row's running
// maximum grows by more than 8 (log2 units); a stale maximum only bounds
// p by 2^8, which fp32 holds exactly enough.
//
// Every wait is bounded in time (globaltimer); a wait that runs out records
// TPLA_ERR_TIMEOUT in the device status word, sets a CTA-wide abort flag so
// all roles stop, and the kernel drains its TMA loads and MMAs before it
// frees tensor memory and returns.
#include "tpla_internal.cuh"
#include "sm100_ptx.cuh"

#include <cuda.h>
#include <mutex>

namespace tpla {
namespace {

using namespace sm100;

constexpr int kThreads = 192;
constexpr int kSoftmaxWarp0 = 2;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

template <int LS, int RD, int NST>
struct Cfg {
    static constexpr int kChunk = 64 * 128;                   // one 64-row x 128-byte swizzled chunk
    static constexpr int kChunksC = LS / 64;
    static constexpr int kChunksK = RD / 64;
    static constexpr int kStageBytes = (kChunksC + kChunksK) * kChunk;
    static constexpr int kK = LS + RD;                         // QK^T contraction length
    static constexpr int kColO = 0;
    static constexpr int kColS = LS;
    static constexpr int kColP = LS + 64;
    static constexpr int kColQ = LS + 96;
    static constexpr int kColsUsed = kColQ + kK / 2;
    static constexpr int kTmemCols = kColsUsed <= 128 ? 128 : (kColsUsed <= 256 ? 256 : 512);
    static constexpr uint32_t kIdescQK = idesc_f16kind(128, 64, false, true);    // bf16 x bf16
    static constexpr uint32_t kIdescPV = idesc_f16kind(128, LS, true, false);    // fp16 x fp16
    static_assert(kColsUsed <= 512, "tensor memory");
    static_assert(LS % 64 == 0 && RD == 64, "tile shape");
};

template <int NST>
struct Bars {
    uint64_t full[NST];
    uint64_t empty[NST];
    uint64_t s_full, s_free, p_full, o_done, q_full, o_free, drain, never;
    uint32_t tmem_base;
    volatile int abort;
};

struct Waiter {
    volatile int* abort;
    unsigned* status;
    uint64_t limit_ns;

    // true when the phase of `parity` completed; false on abort or time-out
    __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = globaltimer_ns();
        for (;;) {
            if (mbar_try_wait(bar, parity)) return true;
            if (*abort) return false;
            if (globaltimer_ns() - t0 > limit_ns) {
                atomicOr(status, kStatusTimeout);
                *abort = 1;
                return false;
            }
        }
    }
};

struct SegFlags {
    bool begin, end;
};

__device__ __forceinline__ SegFlags seg_flags(long long u, long long lo, long long hi, const UnitPos& pos) {
    return {u == lo || pos.tile == 0, u == hi - 1 || pos.tile == pos.ntiles - 1};
}

template <int LS, int RD, int NST>
__global__ void __launch_bounds__(kThreads, 1)
attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_k, Plan p,
                  const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_pe,
                  const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens, Workspace ws,
                  uint64_t wait_ns, int debug_stall) {
    using C = Cfg<LS, RD, NST>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    auto& bars = *reinterpret_cast<Bars<NST>*>(smem + NST * C::kStageBytes);
    const uint32_t stage0 = smem_addr(smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x;

    // every warp derives the same unit range from seq_lens
    const long long U = warp_total_units(seq_lens, p.B, p.max_pages, p.gc);
    if (U == 0) return;
    const long long lo = unit_lo(w, U, p.W), hi = unit_lo(w + 1, U, p.W);
    if (lo >= hi) return;
    const UnitPos pos0 = warp_locate_unit(seq_lens, p.B, p.max_pages, p.gc, lo);

    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_addr(&bars.full[i]), 1);
            mbar_init(smem_addr(&bars.empty[i]), 1);
        }
        mbar_init(smem_addr(&bars.s_full), 1);
        mbar_init(smem_addr(&bars.s_free), 4);
        mbar_init(smem_addr(&bars.p_full), 4);
        mbar_init(smem_addr(&bars.o_done), 1);
        mbar_init(smem_addr(&bars.q_full), 4);
        mbar_init(smem_addr(&bars.o_free), 4);
        mbar_init(smem_addr(&bars.drain), 1);
        mbar_init(smem_addr(&bars.never), 1);
        bars.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(&bars.tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    const Waiter wt{&bars.abort, p.status, wait_ns};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            UnitPos pos = pos0;
            long long j = 0;
            for (long long u = lo; u < hi; ++u, ++j) {
                const int st = (int)(j % NST);
                const uint32_t use = (uint32_t)(j / NST);
                if (use > 0 && !wt.wait(smem_addr(&bars.empty[st]), (use - 1) & 1)) break;
                const int shard = p.shard0 + pos.s;
                const int page = page_lookup(block_table, pos.b, pos.tile, p.max_pages, p.num_pages, p.status);
                // an invalid page reads rows past the end of the tensor: TMA fills zeros
                const int yc = page >= 0 ? (page * p.g + shard) * kPage : p.num_pages * p.g * kPage;
                const int yk = page >= 0 ? page * kPage : p.num_pages * kPage;
                const uint32_t full = smem_addr(&bars.full[st]);
                const uint32_t dst = stage0 + st * C::kStageBytes;
                mbar_arrive_expect_tx(full, C::kStageBytes);
#pragma unroll
                for (int c = 0; c < C::kChunksC; ++c) tma_load_2d(dst + c * C::kChunk, &tm_c, full, c * 64, yc);
                tma_load_2d(dst + C::kChunksC * C::kChunk, &tm_k, full, 0, yk);
                advance_unit(pos, seq_lens, p.B, p.max_pages, p.gc);
            }
            // drain: the last use of every stage must have landed before the CTA exits
            const long long issued = j;
            for (long long t = issued - NST < 0 ? 0 : issued - NST; t < issued; ++t) {
                const int st = (int)(t % NST);
                // bounded wait that ignores the abort flag (the copy is in flight either way)
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(smem_addr(&bars.full[st]), (uint32_t)(t / NST) & 1)) {
                    if (globaltimer_ns() - t0 > wait_ns) {
                        atomicOr(p.status, kStatusTimeout);
                        break;
                    }
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if (debug_stall) ok = wt.wait(smem_addr(&bars.never), 0);   // nothing arrives: exercises the time-out
            UnitPos pos = pos0;
            long long j = 0;
            int seg = -1;
            bool prev_end = true, prev_first = false;
            int prev_seg = -1;
            auto issue_pv = [&](long long t, bool first, int tseg) -> bool {
                if (!wt.wait(smem_addr(&bars.p_full), (uint32_t)(t & 1))) return false;
                if (first && tseg > 0 && !wt.wait(smem_addr(&bars.o_free), (uint32_t)((tseg - 1) & 1))) return false;
                tc_fence_after();
                const uint32_t sb = stage0 + (int)(t % NST) * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    const uint64_t bd = smem_desc_sw128(sb + kk * 2048, C::kChunk, 1024);
                    mma_ts(tmem + C::kColO, tmem + C::kColP + kk * 8, bd, C::kIdescPV, (first && kk == 0) ? 0u : 1u);
                }
                mma_commit(smem_addr(&bars.empty[(int)(t % NST)]));
                mma_commit(smem_addr(&bars.o_done));
                return true;
            };
            for (long long u = lo; ok && u < hi; ++u, ++j) {
                const SegFlags f = seg_flags(u, lo, hi, pos);
                if (f.begin) {
                    ++seg;
                    if (!wt.wait(smem_addr(&bars.q_full), (uint32_t)(seg & 1))) break;
                }
                const int st = (int)(j % NST);
                if (!wt.wait(smem_addr(&bars.full[st]), (uint32_t)((j / NST) & 1))) break;
                if (j > 0 && !wt.wait(smem_addr(&bars.s_free), (uint32_t)((j - 1) & 1))) break;
                tc_fence_after();
                const uint32_t sb = stage0 + st * C::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < C::kK / 16; ++kk) {
                    const uint64_t bd = smem_desc_sw128(sb + (kk >> 2) * C::kChunk + (kk & 3) * 32, 16, 1024);
                    mma_ts(tmem + C::kColS, tmem + C::kColQ + kk * 8, bd, C::kIdescQK, kk > 0 ? 1u : 0u);
                }
                mma_commit(smem_addr(&bars.s_full));
                if (j > 0 && !prev_end && !issue_pv(j - 1, prev_first, prev_seg)) break;
                if (f.end && !issue_pv(j, f.begin, seg)) break;
                prev_end = f.end;
                prev_first = f.begin;
                prev_seg = seg;
                advance_unit(pos, seq_lens, p.B, p.max_pages, p.gc);
            }
            // drain every MMA this thread issued before tensor memory is freed
            mma_commit(smem_addr(&bars.drain));
            const uint64_t t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_addr(&bars.drain), 0)) {
                if (globaltimer_ns() - t0 > wait_ns) {
                    atomicOr(p.status, kStatusTimeout);
                    break;
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax / epilogue (warps 2..5)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;                 // head row == TMEM lane
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const bool warp_active = quad * 32 < p.H;
        const bool row_active = row < p.H;
        const int tid_sm = threadIdx.x - kSoftmaxWarp0 * 32;   // 0..127
        UnitPos pos = pos0;
        long long j = 0;
        long long last_o = -1;                            // last PV whose completion was observed
        float m = -INFINITY, l = 0.f;
        bool first_tile = true;
        auto wait_o = [&](long long t) -> bool {
            if (t <= last_o) return true;
            if (!wt.wait(smem_addr(&bars.o_done), (uint32_t)(t & 1))) return false;
            last_o = t;
            tc_fence_after();
            return true;
        };
        for (long long u = lo; u < hi; ++u, ++j) {
            const SegFlags f = seg_flags(u, lo, hi, pos);
            const int shard = p.shard0 + pos.s;
            if (f.begin) {
                // Q row of this head for (b, shard) into tensor memory: [q~_s | q_pe] as bf16 pairs
                if (warp_active) {
                    const uint4* qs = reinterpret_cast<const uint4*>(q + ((size_t)pos.b * p.H + row) * p.L +
                                                                     (size_t)shard * LS);
                    const uint4* qp = reinterpret_cast<const uint4*>(q_pe + ((size_t)pos.b * p.H + row) * RD);
#pragma unroll
                    for (int c = 0; c < C::kK / 64; ++c) {
                        uint32_t r[32];
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            uint4 x = make_uint4(0, 0, 0, 0);
                            if (row_active) x = c < C::kChunksC ? __ldg(qs + c * 8 + v) : __ldg(qp + (c - C::kChunksC) * 8 + v);
                            r[4 * v + 0] = x.x; r[4 * v + 1] = x.y; r[4 * v + 2] = x.z; r[4 * v + 3] = x.w;
                        }
                        tmem_st32(lane_base + C::kColQ + c * 32, r);
                    }
                    tmem_wait_st();
                }
                (void)effective_len(seq_lens, pos.b, p.max_pages, p.status);
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bars.q_full));
                m = -INFINITY;
                l = 0.f;
                first_tile = true;
            }
            const int valid = min(kPage, pos.T - pos.tile * kPage);
            if (!wt.wait(smem_addr(&bars.s_full), (uint32_t)(j & 1))) break;
            tc_fence_after();
            float s[64];
            if (warp_active) {
                uint32_t r0[32], r1[32];
                tmem_ld32(lane_base + C::kColS, r0);
                tmem_ld32(lane_base + C::kColS + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    s[t] = __uint_as_float(r0[t]);
                    s[t + 32] = __uint_as_float(r1[t]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars.s_free));

            // QK^T of this tile is done with its shared memory: turn the latent rows into the fp16
            // operand of PV, and zero rows past the sequence end so P*C never meets stale bits
            {
                uint8_t* sb = smem + (int)(j % NST) * C::kStageBytes;
#pragma unroll 4
                for (int i = tid_sm; i < C::kChunksC * kPage * 8; i += 128) {
                    const int c = i >> 9, rr = (i >> 3) & 63, seg16 = i & 7;
                    uint4* ptr = reinterpret_cast<uint4*>(sb + c * C::kChunk + rr * 128 + seg16 * 16);
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (rr < valid) {
                        v = *ptr;
                        v.x = bf16x2_to_f16x2(v.x);
                        v.y = bf16x2_to_f16x2(v.y);
                        v.z = bf16x2_to_f16x2(v.z);
                        v.w = bf16x2_to_f16x2(v.w);
                    }
                    *ptr = v;
                }
                fence_proxy_async_smem();
            }

            bool alive = true;
            if (warp_active) {
                float mt = -INFINITY;
#pragma unroll
                for (int t = 0; t < 64; ++t) {
                    s[t] = t < valid ? s[t] * p.scale_log2 : -INFINITY;
                    mt = fmaxf(mt, s[t]);
                }
                if (first_tile) {
                    m = mt;
                } else {
                    const bool need = mt > m + kRescaleThreshold;
                    if (__any_sync(0xffffffffu, need)) {
                        const float m_use = need ? mt : m;
                        const float alpha = exp2f(m - m_use);
                        if (!wait_o(j - 1)) { alive = false; }
                        if (alive) {
#pragma unroll 1
                            for (int c = 0; c < LS / 32; ++c) {
                                uint32_t r[32];
                                tmem_ld32(lane_base + C::kColO + c * 32, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
                                tmem_st32(lane_base + C::kColO + c * 32, r);
                            }
                            tmem_wait_st();
                            l *= alpha;
                            m = m_use;
                        }
                    }
                }
            }
            if (!alive) break;
            uint32_t pk[32];
            if (warp_active) {
                float ls = 0.f;
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const float e0 = exp2f(s[2 * t] - m), e1 = exp2f(s[2 * t + 1] - m);
                    ls += e0 + e1;
                    pk[t] = pack_f16x2(e0, e1);
                }
                l += ls;
            }
            // the single P buffer is free once PV of the previous tile has completed
            if (j > 0 && !wait_o(j - 1)) break;
            if (warp_active) {
                tmem_st32(lane_base + C::kColP, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&bars.p_full));
            first_tile = false;

            if (f.end) {
                if (!wait_o(j)) break;
                const long long seg_first = (u - pos.tile) < lo ? lo : (u - pos.tile);
                const int slot = seg_first == lo ? w : p.W + pos.b * p.gc + pos.s;
                if (warp_active) {
                    const float inv_l = 1.0f / l;
                    float4* dst = reinterpret_cast<float4*>(ws.part_o + ((size_t)slot * p.H + row) * LS);
#pragma unroll 1
                    for (int c = 0; c < LS / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + C::kColO + c * 32, r);
                        tmem_wait_ld();
                        if (row_active) {
#pragma unroll
                            for (int v = 0; v < 8; ++v)
                                dst[c * 8 + v] = make_float4(__uint_as_float(r[4 * v]) * inv_l,
                                                             __uint_as_float(r[4 * v + 1]) * inv_l,
                                                             __uint_as_float(r[4 * v + 2]) * inv_l,
                                                             __uint_as_float(r[4 * v + 3]) * inv_l);
                        }
                    }
                    if (row_active) ws.part_lse[(size_t)slot * p.H + row] = m + log2f(l);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bars.o_free));
            }
            advance_unit(pos, seq_lens, p.B, p.max_pages, p.gc);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D bf16 tensor map over [rows][cols] with a 64 x 64 box and 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows) {
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

template <int LS, int RD, int NST>
cudaError_t launch_t(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe, const __nv_bfloat16* ckv,
                     const __nv_bfloat16* kpe, const int32_t* bt, const int32_t* seq_lens, Workspace ws,
                     uint64_t wait_ns, int debug_stall, cudaStream_t stream) {
    using C = Cfg<LS, RD, NST>;
    CUtensorMap tc, tk;
    if (!make_map(&tc, ckv, LS, (uint64_t)p.num_pages * p.g * kPage)) return cudaErrorInvalidValue;
    if (!make_map(&tk, kpe, RD, (uint64_t)p.num_pages * kPage)) return cudaErrorInvalidValue;
    const size_t smem = 1024 + (size_t)NST * C::kStageBytes + sizeof(Bars<NST>);
    static_assert(C::kTmemCols < 512 || (1024 + NST * C::kStageBytes) > 116 * 1024,
                  "a 512-column TMEM allocation needs one CTA per SM");
    auto kern = attn_sm100_kernel<LS, RD, NST>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    kern<<<p.W, kThreads, smem, stream>>>(tc, tk, p, q, q_pe, bt, seq_lens, ws, wait_ns, debug_stall);
    return cudaGetLastError();
}

}  // namespace

bool sm100_supports(const Plan& p) {
    return p.R == 64 && (p.Ls == 64 || p.Ls == 128 || p.Ls == 256);
}

cudaError_t launch_attention_sm100(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                   const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                   const int32_t* block_table, const int32_t* seq_lens, Workspace ws,
                                   int wait_limit_us, int debug_stall, cudaStream_t stream) {
    const uint64_t wait_ns = (wait_limit_us > 0 ? (uint64_t)wait_limit_us : 1000000ull) * 1000ull;
    switch (p.Ls) {
        case 256: return launch_t<256, 64, 5>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, wait_ns, debug_stall, stream);
        case 128: return launch_t<128, 64, 8>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, wait_ns, debug_stall, stream);
        case 64: return launch_t<64, 64, 12>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, wait_ns, debug_stall, stream);
    }
    return cudaErrorNotSupported;
}

}  // namespace tpla
