// tcgen05 / TMEM / TMA split-KV attention for 512 latent columns per shard (g = 1 at
// kv_lora_rank 512: MLA decode in absorbed form), for sm_100a (B200).
//
// What it computes (TPLA paper, Abstract: TPLA with one shard is MLA, and TPLA is drop-in for MLA):
// for every shard s of the call and every head h of sequence b
//     z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t),   o_{h,s} = sum_t softmax_t(z) c_{t,s}
// as an online softmax over the tiles of one split-KV segment (schedule in tpla_internal.cuh),
// leaving the normalised o and the log2-sum-exp per head for the combine kernel.
//
// Why a CTA pair.  With 128 heads as the MMA M dimension, O alone is 128 x 512 fp32: all of one
// SM's tensor memory.  So each split-KV worker is two CTAs (blockIdx.y = 0, 1); CTA c keeps the
// output columns [256c, 256c + 256).  Both CTAs load the whole 64-token page (the second read of
// the pair is served by L2) and compute the same full score tile
//     S[h, t] = Q[h, :] . [C_s | K_pe][t, :]^T        M = 128, N = 64, K = 512 + 64
// (the MMAs are deterministic, so both CTAs hold bit-identical S, softmax state and row sums; CTA 0
// alone writes the log-sum-exps), then
//     O_c[h, :] += P[h, t] . C_s[t, 256c : 256c + 256]  M = 128, N = 256, K = 64
// Splitting the tokens instead would need the partial scores of both CTAs added before the
// softmax; splitting the columns needs no exchange at all.
//
// Operand placement (tensor memory: 512 columns of 128 lanes):
//   tensor memory: O_c (256 columns), S (64), and query latent columns 0-383 as bf16 pairs (192),
//                  the A operand of the first 24 QK^T steps (A from tensor memory runs at about
//                  twice the rate of A from shared memory on B200);
//   shared memory: query latent columns 384-511 and the RoPE query (three 128-row chunks, the A
//                  operand of the last 12 QK^T steps), P (A operand of PV), and two pipeline stages
//                  of one page each: 8 latent chunks + 1 RoPE chunk of 64 rows x 128 B, 128B-swizzled,
//                  the K-major B operand of QK^T and (chunks 4c..4c+3) the MN-major B operand of PV.
//
// Precision: as in attn_sm100.cu -- QK^T multiplies the bf16 inputs as they are; a tile of a
// sequence shorter than kExactPVBelow tokens runs PV in fp16 (its PV chunks converted in place,
// scaled by the power of two the softmax warps agree on, P scaled by its inverse), otherwise in
// bf16; rows past the end of the sequence are zeroed before PV reads them.
//
// Warp roles (320 threads): warp 0 issues the TMA loads, warp 1 allocates tensor memory and issues
// the MMAs from one thread, warps 2-9 are two softmax warpgroups over all 128 rows (one head per
// thread), each taking 32 of the tile's 64 score columns and, at the end of a segment, 128 of the
// CTA's 256 output columns.  The epilogue stages the normalised rows in the shared-memory query
// region (free once the segment's last QK^T has completed) and writes them with TMA stores; the
// next segment's query is loaded after that.  Every wait is bounded (TPLA_ERR_TIMEOUT in the device
// status word, a CTA-wide abort, loads and MMAs drained, tensor memory freed).
#include "tpla_internal.cuh"
#include "sm100_ptx.cuh"
#include "attn_sm100_common.cuh"

namespace tpla {
namespace {

using namespace sm100;

constexpr int kThreads = 320;
constexpr int kSoftmaxWarp0 = 2;
constexpr int kSoftmaxWarps = 8;
constexpr int kLs = 512;                       // latent columns per shard
constexpr int kRd = 64;                        // RoPE width
constexpr int kNst = 2;                        // pipeline stages
constexpr int kTok = kPage;                    // tokens per tile: one page
constexpr float kRescaleThreshold = 8.0f;      // log2 units
constexpr int kExactPVBelow = 8192;            // sequences shorter than this may run PV in fp16
constexpr int kPageAhead = 4;                  // page-table entries the producer loads ahead

constexpr int kChunk = kTok * 128;             // one 64-column slice of the page: 64 rows x 128 B
constexpr int kChunksC = kLs / 64;             // 8 latent chunks
constexpr int kStageBytes = (kChunksC + 1) * kChunk;      // + the RoPE chunk: 72 KB
constexpr int kQtDims = 384;                   // query latent columns held in tensor memory
constexpr int kQsChunk = 128 * 128;            // a 128-row x 128 B query chunk in shared memory
constexpr int kQsChunks = (kLs - kQtDims) / 64 + 1;       // 2 latent + 1 RoPE
constexpr int kPBytes = 128 * kTok * 2;        // P: 128 rows x 64 tokens bf16
constexpr int kColO = 0;                       // 256 columns
constexpr int kColS = 256;                     // 64 columns
constexpr int kColQ = 320;                     // 192 columns
constexpr int kTmemCols = 512;
constexpr int kStepsT = kQtDims / 16;          // QK^T steps with A in tensor memory
constexpr int kStepsS = (kLs - kQtDims) / 16;  // ... with A (latent) in shared memory
constexpr int kStepsR = kRd / 16;              // ... over the RoPE key
constexpr uint32_t kIdescQK = idesc_f16kind(128, kTok, false, true);
constexpr uint32_t kIdescPVf16 = idesc_f16kind(128, 256, true, false);
constexpr uint32_t kIdescPVbf16 = idesc_f16kind(128, 256, true, true);
constexpr int kCvt = 4 * kTok * 8 / (kSoftmaxWarps * 32);   // 16-byte pieces of the CTA's PV chunks per thread
constexpr size_t kSmem = 1024 + (size_t)kNst * kStageBytes + (size_t)kQsChunks * kQsChunk + kPBytes;
static_assert(kColQ + kQtDims / 2 == kTmemCols, "tensor memory");
static_assert(kQsChunks * kQsChunk >= kSoftmaxWarps * 4096, "epilogue staging fits the query region");
static_assert(kCvt == 8, "conversion split");

struct Bars {
    uint64_t full[kNst];
    uint64_t empty[kNst];
    uint64_t s_full, s_free, p_full, o_done;
    uint64_t q_full, o_free, xmax, xsum, drain, never, vote, epi;
    float xmax_buf[2][2][128];     // [tile parity][warpgroup][row]
    float xsum_buf[2][2][128];     // [segment parity][warpgroup][row]
    uint32_t vote_max[2][8];       // [tile parity][softmax warp]: largest |latent| bit pattern seen
    int pv_f16[2];                 // [tile parity]: PV of that tile runs in fp16
    uint32_t tmem_base;
    volatile int abort;
};
static_assert(kSmem + sizeof(Bars) <= 227 * 1024, "shared memory");

__global__ void __launch_bounds__(kThreads, 1)
attn_wide_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_o, Plan p,
                 const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_pe,
                 const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens, Workspace ws,
                 uint64_t wait_ns, int debug_stall) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* qs_smem = smem + kNst * kStageBytes;            // query chunks: latent 384-447, 448-511, RoPE
    uint8_t* p_smem = qs_smem + kQsChunks * kQsChunk;        // P
    auto& bars = *reinterpret_cast<Bars*>(p_smem + kPBytes);
    const uint32_t stage0 = smem_addr(smem);
    const uint32_t qs_addr = smem_addr(qs_smem);
    const uint32_t p_addr = smem_addr(p_smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x;
    const int half = blockIdx.y;                              // output columns [256 half, 256 half + 256)

    if (threadIdx.x == 0) {
        for (int i = 0; i < kNst; ++i) {
            mbar_init(smem_addr(&bars.full[i]), 1);
            mbar_init(smem_addr(&bars.empty[i]), 1);
        }
        mbar_init(smem_addr(&bars.s_full), 1);
        mbar_init(smem_addr(&bars.s_free), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.p_full), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.o_done), 1);
        mbar_init(smem_addr(&bars.q_full), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.o_free), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.xmax), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.xsum), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.drain), 1);
        mbar_init(smem_addr(&bars.never), 1);
        mbar_init(smem_addr(&bars.vote), kSoftmaxWarps);
        mbar_init(smem_addr(&bars.epi), kSoftmaxWarps);
        bars.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tensor_map(&tm_c);
        prefetch_tensor_map(&tm_k);
    }
    // every input may have been written by the previous kernel on the stream: wait for it
    pdl_wait();

    const long long V = warp_total_weight(seq_lens, p);
    if (V == 0) return;
    const long long lo = warp_unit_at_weight(seq_lens, p, unit_lo(w, V, p.W));
    const long long hi = warp_unit_at_weight(seq_lens, p, unit_lo(w + 1, V, p.W));
    if (lo >= hi) {
        // a worker with no units leaves a zero-weight partial in its slot (see attn_sm100.cu)
        if (half == 0)
            for (int i = threadIdx.x; i < p.H; i += blockDim.x) ws.part_lse[(size_t)w * p.H + i] = -INFINITY;
        return;
    }
    const UnitPos pos0 = warp_locate_unit(seq_lens, p.B, p.max_pages, p.gc, lo);

    if (warp == 1) {
        tmem_alloc(smem_addr(&bars.tmem_base), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    const Waiter wt{&bars.abort, p.status, wait_ns * 2};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            UnitPos ahead = pos0;
            long long ua = lo;
            auto raw_page = [&](const UnitPos& u) -> int {
                return block_table ? __ldg(block_table + (size_t)u.b * p.max_pages + u.tile)
                                   : u.b * p.max_pages + u.tile;
            };
            int pg[kPageAhead];
#pragma unroll
            for (int k = 0; k < kPageAhead; ++k) {
                pg[k] = -1;
                if (ua < hi) {
                    pg[k] = raw_page(ahead);
                    advance_unit(ahead, seq_lens, p.B, p.max_pages, p.gc);
                    ++ua;
                }
            }
            Tile t = make_tile(pos0, lo, lo, hi, 1);
            long long j = 0;
            for (; t.u < hi; ++j) {
                const int st = (int)(j % kNst);
                const uint32_t use = (uint32_t)(j / kNst);
                // every popped entry belongs to a unit of the range; one outside [0, num_pages) is a
                // caller error, recorded, and the page reads as zeros
                int page = pg[0];
                if (page < 0 || page >= p.num_pages) {
                    atomicOr(p.status, kStatusIndex);
                    page = -1;
                }
#pragma unroll
                for (int k = 0; k + 1 < kPageAhead; ++k) pg[k] = pg[k + 1];
                pg[kPageAhead - 1] = -1;
                if (ua < hi) {
                    pg[kPageAhead - 1] = raw_page(ahead);
                    advance_unit(ahead, seq_lens, p.B, p.max_pages, p.gc);
                    ++ua;
                }
                if (use > 0 && !wt.wait(smem_addr(&bars.empty[st]), (use - 1) & 1)) break;
                const int shard = p.shard0 + t.pos.s;
                if (t.begin && j > 0) {
                    // the next segment's query is loaded after this segment's epilogue: have it in L2
                    const __nv_bfloat16* qrow = q + (size_t)t.pos.b * p.H * p.L + (size_t)shard * kLs;
                    for (int h = 0; h < p.H; ++h) prefetch_l2(qrow + (size_t)h * p.L, kLs * 2);
                    prefetch_l2(q_pe + (size_t)t.pos.b * p.H * kRd, (uint32_t)(p.H * kRd * 2));
                }
                const uint32_t full = smem_addr(&bars.full[st]);
                const uint32_t dst = stage0 + st * kStageBytes;
                mbar_arrive_expect_tx(full, kStageBytes);
                // a missing or invalid page reads rows past the end of the tensor: TMA fills zeros
                const int yc = page >= 0 ? (page * p.g + shard) * kPage : p.num_pages * p.g * kPage;
                const int yk = page >= 0 ? page * kPage : p.num_pages * kPage;
#pragma unroll
                for (int c = 0; c < kChunksC; ++c) tma_load_2d(dst + c * kChunk, &tm_c, full, c * 64, yc);
                tma_load_2d(dst + kChunksC * kChunk, &tm_k, full, 0, yk);
                t = next_tile(t, seq_lens, p, lo, hi);
            }
            pdl_trigger();
            // drain: the last use of every stage must have landed before the CTA exits
            for (long long x = j - kNst < 0 ? 0 : j - kNst; x < j; ++x) {
                const int st = (int)(x % kNst);
                const uint64_t t0 = globaltimer_ns();
                while (!mbar_try_wait(smem_addr(&bars.full[st]), (uint32_t)(x / kNst) & 1)) {
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
            // Whichever MMA is ready goes first, PV of the oldest tile ahead of QK^T of the next one
            // (it releases a stage); each stream has its own tile cursor.
            Tile tq = make_tile(pos0, lo, lo, hi, 1), tv = tq;
            long long jq = 0, jv = 0;
            int qseg = -1, vseg = -1;
            bool vbegun = false;
            long long idle_since = clock64();
            while (ok && tv.u < hi) {
                bool did = false;
                if (jv < jq) {
                    if (tv.begin && !vbegun) {
                        ++vseg;
                        vbegun = true;
                    }
                    if (mbar_test_wait(smem_addr(&bars.p_full), (uint32_t)(jv & 1)) &&
                        (!tv.begin || vseg == 0 ||
                         mbar_test_wait(smem_addr(&bars.o_free), (uint32_t)((vseg - 1) & 1)))) {
                        tc_fence_after();
                        const int st = (int)(jv % kNst);
                        const uint32_t sb = stage0 + st * kStageBytes + half * 4 * kChunk;
                        const uint32_t idesc_pv = bars.pv_f16[jv & 1] ? kIdescPVf16 : kIdescPVbf16;
#pragma unroll
                        for (int kk = 0; kk < kTok / 16; ++kk) {
                            // A: 16 tokens of P (K-major); B: the same 16 token rows of this CTA's four
                            // latent chunks (MN-major, chunk stride 8 KB)
                            const uint64_t ad = smem_desc_sw128(p_addr + kk * 32, 16, 1024);
                            const uint64_t bd = smem_desc_sw128(sb + kk * 2048, kChunk, 1024);
                            mma_ss(tmem + kColO, ad, bd, idesc_pv, (tv.begin && kk == 0) ? 0u : 1u);
                        }
                        mma_commit(smem_addr(&bars.empty[st]));
                        mma_commit(smem_addr(&bars.o_done));
                        tv = next_tile(tv, seq_lens, p, lo, hi);
                        ++jv;
                        vbegun = false;
                        did = true;
                    }
                }
                if (tq.u < hi) {
                    const int st = (int)(jq % kNst);
                    if ((!tq.begin || mbar_test_wait(smem_addr(&bars.q_full), (uint32_t)((qseg + 1) & 1))) &&
                        mbar_test_wait(smem_addr(&bars.full[st]), (uint32_t)((jq / kNst) & 1)) &&
                        (jq == 0 || mbar_test_wait(smem_addr(&bars.s_free), (uint32_t)((jq - 1) & 1)))) {
                        if (tq.begin) ++qseg;
                        tc_fence_after();
                        const uint32_t sb = stage0 + st * kStageBytes;
                        const uint32_t d = tmem + kColS;
#pragma unroll
                        for (int kk = 0; kk < kStepsT; ++kk) {
                            const uint64_t bd = smem_desc_sw128(sb + (kk >> 2) * kChunk + (kk & 3) * 32, 16, 1024);
                            mma_ts(d, tmem + kColQ + kk * 8, bd, kIdescQK, kk > 0 ? 1u : 0u);
                        }
#pragma unroll
                        for (int kk = 0; kk < kStepsS + kStepsR; ++kk) {
                            // query chunk kk/4 (latent 384-447, 448-511, then RoPE) against stage chunk
                            // 6 + kk/4 (latent 384-447, 448-511, then the RoPE key)
                            const uint64_t ad = smem_desc_sw128(qs_addr + (kk >> 2) * kQsChunk + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd =
                                smem_desc_sw128(sb + (kStepsT / 4 + (kk >> 2)) * kChunk + (kk & 3) * 32, 16, 1024);
                            mma_ss(d, ad, bd, kIdescQK, 1u);
                        }
                        mma_commit(smem_addr(&bars.s_full));
                        tq = next_tile(tq, seq_lens, p, lo, hi);
                        ++jq;
                        did = true;
                    }
                }
                if (did) {
                    idle_since = clock64();
                } else {
                    if (bars.abort) break;
                    if ((uint64_t)(clock64() - idle_since) > wt.limit_cycles) {
                        atomicOr(p.status, kStatusTimeout);
                        bars.abort = 1;
                        break;
                    }
                }
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
        // ------------------------------------------------------------ softmax / epilogue (warps 2..9)
        const int sw = warp - kSoftmaxWarp0;              // 0..7
        const int wg = sw >> 2;                           // score columns [32 wg, 32 wg + 32), O columns [128 wg, +128)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;                 // TMEM lane: head
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        const bool warp_active = quad * 32 < p.H;
        const bool row_active = row < p.H;
        const int tid_sm = threadIdx.x - kSoftmaxWarp0 * 32;   // 0..255
        const float sc = fabsf(p.scale_log2);
        const uint32_t qflip = p.scale_log2 < 0.f ? 0x80008000u : 0u;   // negative scale: flip the query's sign
        constexpr int kCols = kTok / 2;                   // score columns per thread: 32
        const int cbase = wg * kCols;
        long long last_o = -1;
        int seg = -1;
        float m = -INFINITY, l = 0.f;
        bool first_tile = true;
        bool exact = false;
        long long nvote = 0;
        auto wait_o = [&](long long t) -> bool {
            if (t <= last_o) return true;
            if (!wt.wait(smem_addr(&bars.o_done), (uint32_t)(t & 1))) return false;
            last_o = t;
            tc_fence_after();
            return true;
        };
        // Query of one (b, shard) segment: latent columns 0-383 into tensor memory as bf16 pairs
        // (the warpgroups take alternate 64-column chunks), columns 384-511 and the RoPE query into
        // the three shared-memory chunks (warpgroup wg writes the 16-byte pieces 4wg..4wg+3 of each).
        auto load_q = [&](const UnitPos& qp) {
            const int shard = p.shard0 + qp.s;
            if (warp_active) {
                const uint4* qs = reinterpret_cast<const uint4*>(q + ((size_t)qp.b * p.H + row) * p.L +
                                                                 (size_t)shard * kLs);
                const uint4* qpp = reinterpret_cast<const uint4*>(q_pe + ((size_t)qp.b * p.H + row) * kRd);
                // shared-memory part first (12 loads), then the tensor-memory chunks one at a time, so
                // that no more than 12 + 8 loads are held in registers
                uint4 y[3][4];
#pragma unroll
                for (int i = 0; i < 3; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        y[i][k] = !row_active ? make_uint4(0, 0, 0, 0)
                                  : i < 2     ? __ldg(qs + (kQtDims / 8) + i * 8 + wg * 4 + k)
                                              : __ldg(qpp + wg * 4 + k);
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int c = wg + 2 * i;             // tensor-memory chunk (64 columns)
                    uint4 x[8];
#pragma unroll
                    for (int v = 0; v < 8; ++v) x[v] = row_active ? __ldg(qs + c * 8 + v) : make_uint4(0, 0, 0, 0);
                    if (i == 0) {
#pragma unroll
                        for (int ii = 0; ii < 3; ++ii)
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                *reinterpret_cast<uint4*>(qs_smem + ii * kQsChunk + sw128_offset(row, wg * 4 + k)) =
                                    make_uint4(y[ii][k].x ^ qflip, y[ii][k].y ^ qflip, y[ii][k].z ^ qflip,
                                               y[ii][k].w ^ qflip);
                    }
                    uint32_t r[32];
#pragma unroll
                    for (int v = 0; v < 8; ++v) {
                        r[4 * v + 0] = x[v].x ^ qflip; r[4 * v + 1] = x[v].y ^ qflip;
                        r[4 * v + 2] = x[v].z ^ qflip; r[4 * v + 3] = x[v].w ^ qflip;
                    }
                    tmem_st32(lane_base + kColQ + c * 32, r);
                }
                tmem_wait_st();
            } else {
                // rows past H: zero query in shared memory (their tensor-memory rows only feed S rows
                // that are never read)
#pragma unroll
                for (int i = 0; i < 3; ++i)
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        *reinterpret_cast<uint4*>(qs_smem + i * kQsChunk + sw128_offset(row, wg * 4 + k)) =
                            make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(smem_addr(&bars.q_full));
        };
        Tile t = make_tile(pos0, lo, lo, hi, 1);
        load_q(pos0);
        long long j = 0;
        for (; t.u < hi; ++j) {
            const UnitPos pos = t.pos;
            if (t.begin) {
                ++seg;
                if (wg == 0 && lane == 0 && half == 0) (void)effective_len(seq_lens, pos.b, p.max_pages, p.status);
                m = -INFINITY;
                l = 0.f;
                first_tile = true;
                exact = pos.T < kExactPVBelow;
            }
            const int valid = min(kTok, pos.T - pos.tile * kPage);
            const bool tail = valid < kTok;
            if (!wt.wait(smem_addr(&bars.s_full), (uint32_t)(j & 1))) break;
            tc_fence_after();
            float s[kCols];
            if (warp_active) {
                uint32_t r[32];
                tmem_ld32(lane_base + kColS + cbase, r);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < 32; ++k) s[k] = __uint_as_float(r[k]);
            } else {
#pragma unroll
                for (int k = 0; k < kCols; ++k) s[k] = 0.f;
            }
            tc_fence_before();
            warp_arrive(smem_addr(&bars.s_free));
            uint8_t* sb = smem + (int)(j % kNst) * kStageBytes;

            float ext = -INFINITY;
            if (warp_active) {
                if (tail) {
#pragma unroll
                    for (int k = 0; k < kCols; ++k) s[k] = cbase + k < valid ? s[k] : -INFINITY;
                }
                float e4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) e4[k] = s[k];
#pragma unroll
                for (int k = 4; k < kCols; ++k) e4[k & 3] = fmaxf(e4[k & 3], s[k]);
                ext = fmaxf(fmaxf(e4[0], e4[1]), fmaxf(e4[2], e4[3]));
            }
            // reference maximum of this tile's exponentials (see attn_sm100.cu): the running
            // maximum, raised to this warpgroup's own when that exceeds it by more than the threshold
            const float m_loc = ext * sc;
            const bool raise = warp_active && m_loc > -INFINITY && (first_tile || m_loc > m + kRescaleThreshold);
            const float m_ref = raise ? m_loc : (m > -INFINITY ? m : 0.f);
            bars.xmax_buf[j & 1][wg][row] = raise ? m_loc : -INFINITY;
            warp_arrive(smem_addr(&bars.xmax));
            // PV type of this tile (pv_fp16_shift): fp16 for a short segment, scaled by a power of two
            // chosen from the largest |value| of this CTA's PV chunks over the valid rows
            bool f16 = false;
            float cshift = 1.f, pshift = 1.f;             // 2^e for the latent tile, 2^-e for P
            if (exact) {
                uint32_t mx = 0;
#pragma unroll
                for (int k = 0; k < kCvt; ++k) {
                    const int i = tid_sm + k * kSoftmaxWarps * 32;
                    const int rr = (i >> 3) & (kTok - 1);
                    if (rr < valid) {
                        const uint4 v = *reinterpret_cast<const uint4*>(sb + (half * 4 + (i >> 9)) * kChunk + rr * 128 +
                                                                        (i & 7) * 16);
                        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                                                  __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
                    }
                }
                mx = __reduce_max_sync(0xffffffffu, max(mx & 0xFFFFu, mx >> 16));
                if (lane == 0) bars.vote_max[nvote & 1][sw] = mx;
                warp_arrive(smem_addr(&bars.vote));
            }
            uint32_t pk[kCols / 2];
            float lt = 0.f;
            auto pack = [&]() {
                if (f16) {
#pragma unroll
                    for (int k = 0; k < kCols / 2; ++k) pk[k] = pack_f16x2(s[2 * k] * pshift, s[2 * k + 1] * pshift);
                } else {
#pragma unroll
                    for (int k = 0; k < kCols / 2; ++k) pk[k] = pack_bf16x2(s[2 * k], s[2 * k + 1]);
                }
            };
            if (warp_active) {
                const float nm = -m_ref;
#pragma unroll
                for (int k = 0; k < kCols; ++k) s[k] = ex2_approx(fmaf(s[k], sc, nm));
                if (tail) {
#pragma unroll
                    for (int k = 0; k < kCols; ++k) s[k] = cbase + k < valid ? s[k] : 0.f;
                }
                float l4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int k = 0; k < kCols; ++k) l4[k & 3] += s[k];
                lt = (l4[0] + l4[1]) + (l4[2] + l4[3]);
            }
            if (exact) {
                if (!wt.wait(smem_addr(&bars.vote), (uint32_t)(nvote & 1))) break;
                uint32_t tmax = 0;
#pragma unroll
                for (int k = 0; k < kSoftmaxWarps; ++k) tmax = max(tmax, bars.vote_max[nvote & 1][k]);
                ++nvote;
                int e = 0;
                f16 = pv_fp16_shift(tmax, e);
                cshift = __int_as_float((127 + e) << 23);
                pshift = __int_as_float((127 - e) << 23);
            }
            if (warp_active) {
                pack();
            } else {
#pragma unroll
                for (int k = 0; k < kCols / 2; ++k) pk[k] = 0u;
            }
            if (f16) {
                // this CTA's PV chunks -> fp16 in place (rows past the sequence end -> 0)
#pragma unroll
                for (int k = 0; k < kCvt; ++k) {
                    const int i = tid_sm + k * kSoftmaxWarps * 32;
                    const int rr = (i >> 3) & (kTok - 1);
                    uint4* ptr = reinterpret_cast<uint4*>(sb + (half * 4 + (i >> 9)) * kChunk + rr * 128 + (i & 7) * 16);
                    uint4 v = *ptr;
                    if (rr < valid) {
                        v.x = bf16x2_to_f16x2_scaled(v.x, cshift);
                        v.y = bf16x2_to_f16x2_scaled(v.y, cshift);
                        v.z = bf16x2_to_f16x2_scaled(v.z, cshift);
                        v.w = bf16x2_to_f16x2_scaled(v.w, cshift);
                    } else {
                        v = make_uint4(0, 0, 0, 0);
                    }
                    *ptr = v;
                }
            } else if (tail) {
                // bf16 kept; the rows past the sequence end of this CTA's PV chunks are zeroed
                const int rows = kTok - valid;
                for (int i = tid_sm; i < 4 * rows * 8; i += kSoftmaxWarps * 32) {
                    const int c = half * 4 + i / (rows * 8), rr = valid + (i / 8) % rows, seg16 = i % 8;
                    *reinterpret_cast<uint4*>(sb + c * kChunk + rr * 128 + seg16 * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            if (!wt.wait(smem_addr(&bars.xmax), (uint32_t)(j & 1))) break;
            {
                const float other = bars.xmax_buf[j & 1][wg ^ 1][row];
                const float m_new = fmaxf(m, fmaxf(raise ? m_loc : -INFINITY, other));
                bool alive = true;
                if (warp_active) {
                    if (__any_sync(0xffffffffu, m_new > m_ref)) {   // P was formed against a lower reference
                        const float f = m_new > m_ref ? ex2_approx(m_ref - m_new) : 1.0f;
#pragma unroll
                        for (int k = 0; k < kCols; ++k) s[k] *= f;
                        lt *= f;
                        pack();
                    }
                    if (!first_tile && __any_sync(0xffffffffu, m_new > m)) {   // O and l were against m
                        const float alpha = m_new > m ? ex2_approx(m - m_new) : 1.0f;
                        if (!wait_o(j - 1)) {
                            alive = false;
                        } else {
#pragma unroll 1
                            for (int c = 0; c < 4; ++c) {
                                const uint32_t ta = lane_base + kColO + wg * 128 + c * 32;
                                uint32_t r[32];
                                tmem_ld32(ta, r);
                                tmem_wait_ld();
#pragma unroll
                                for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * alpha);
                                tmem_st32(ta, r);
                            }
                            tmem_wait_st();
                            l *= alpha;
                        }
                    }
                    m = m_new;
                    l += lt;
                }
                if (!alive) break;
            }
            // the P buffer is free once PV(j - 1), its last reader, has completed
            if (j >= 1 && !wait_o(j - 1)) break;
#pragma unroll
            for (int k = 0; k < kCols / 8; ++k)
                *reinterpret_cast<uint4*>(p_smem + sw128_offset(row, wg * 4 + k)) =
                    make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            if (tid_sm == 0) bars.pv_f16[j & 1] = f16 ? 1 : 0;   // read by the issuer after p_full
            fence_proxy_async_smem();
            warp_arrive(smem_addr(&bars.p_full));
            first_tile = false;

            const Tile tn = next_tile(t, seq_lens, p, lo, hi);
            if (t.end) {
                if (!wait_o(j)) break;
                bars.xsum_buf[seg & 1][wg][row] = l;
                warp_arrive(smem_addr(&bars.xsum));
                if (!wt.wait(smem_addr(&bars.xsum), (uint32_t)(seg & 1))) break;
                const float lsum = l + bars.xsum_buf[seg & 1][wg ^ 1][row];
                const long long u_first = t.u - pos.tile;
                const int slot = u_first >= lo ? p.W + pos.b * p.gc + pos.s : w;
                if (warp_active) {
                    // normalised rows out 32 columns at a time, staged (128B-swizzled) in this warp's
                    // 4 KB of the query region -- free: the segment's last QK^T has completed -- and
                    // written by TMA stores of 32 x 32 boxes; rows past H are clipped by the map
                    const float inv_l = 1.0f / lsum;
                    uint8_t* stile = qs_smem + sw * 4096;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + kColO + wg * 128 + c * 32, r);
                        tmem_wait_ld();
                        if (c > 0) {
                            if (lane == 0) bulk_wait_read_all();
                            __syncwarp();
                        }
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            *reinterpret_cast<float4*>(stile + sw128_offset(lane, v)) =
                                make_float4(__uint_as_float(r[4 * v]) * inv_l, __uint_as_float(r[4 * v + 1]) * inv_l,
                                            __uint_as_float(r[4 * v + 2]) * inv_l, __uint_as_float(r[4 * v + 3]) * inv_l);
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&tm_o, smem_addr(stile), half * 256 + wg * 128 + c * 32, quad * 32, slot);
                            bulk_commit();
                        }
                    }
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    if (row_active && wg == 0 && half == 0) ws.part_lse[(size_t)slot * p.H + row] = m + log2f(lsum);
                }
                tc_fence_before();
                warp_arrive(smem_addr(&bars.o_free));
                if (tn.u < hi) {
                    // every warp's stores have read the query region before the next query overwrites it
                    warp_arrive(smem_addr(&bars.epi));
                    if (!wt.wait(smem_addr(&bars.epi), (uint32_t)(seg & 1))) break;
                    load_q(tn.pos);
                }
            }
            t = tn;
        }
    }

    if (warp >= kSoftmaxWarp0 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace

bool sm100_wide_supports(const Plan& p) { return p.R == kRd && p.Ls == kLs; }

cudaError_t launch_attention_sm100_wide(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe,
                                        const __nv_bfloat16* ckv, const __nv_bfloat16* kpe,
                                        const int32_t* block_table, const int32_t* seq_lens, Workspace ws,
                                        int wait_limit_us, int debug_stall, cudaStream_t stream) {
    if (!sm100_wide_supports(p)) return cudaErrorNotSupported;
    const uint64_t wait_ns = (wait_limit_us > 0 ? (uint64_t)wait_limit_us : 1000000ull) * 1000ull;
    CUtensorMap tc, tk, to;
    if (!make_map(&tc, ckv, kLs, (uint64_t)p.num_pages * p.g * kPage)) return cudaErrorInvalidValue;
    if (!make_map(&tk, kpe, kRd, (uint64_t)p.num_pages * kPage)) return cudaErrorInvalidValue;
    if (!make_map_o(&to, ws.part_o, kLs, p.H, (uint64_t)num_slots(p))) return cudaErrorInvalidValue;
    const size_t smem = kSmem + sizeof(Bars);
    static unsigned long long attr_done = 0;
    cudaError_t e = set_smem_once(attn_wide_kernel, smem, &attr_done);
    if (e != cudaSuccess) return e;
    return launch_pdl(attn_wide_kernel, dim3(p.W, 2), dim3(kThreads), smem, stream, tc, tk, to, p, q, q_pe,
                      block_table, seq_lens, ws, wait_ns, debug_stall);
}

}  // namespace tpla
