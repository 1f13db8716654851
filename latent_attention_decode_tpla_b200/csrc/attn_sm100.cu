// tcgen05 / TMEM / TMA split-KV attention over the shard-contiguous latent
// cache, for sm_100a (B200).
//
// What it computes (TPLA paper, Abstract; edgentiq blog "How TPLA Works"):
// for every shard s of sequence b and every head h
//     z_t = scale * (q~_h[s-slice] . c_{t,s} + q_pe_h . k_pe_t)
//     o_{h,s} = sum_t softmax_t(z) c_{t,s}
// as an online softmax over the tiles of one split-KV segment (schedule in
// tpla_internal.cuh); the result per segment is the normalised o and the
// log2-sum-exp per head, merged later by the combine kernels.
//
// All heads of a sequence share every cache row, so both contractions are
// dense with the heads as the MMA M dimension (M = 128; fewer heads are
// padded).  A tile is two consecutive 64-token pages of one segment (one page
// where a segment has an odd number of pages left; the other half is then
// zero-filled by TMA and masked):
//     S[h, t]  = Q[h, :] . [C_s | K_pe][t, :]^T     M=128, N=128, K=Ls+R
//     O[h, :] += P[h, t] . C_s[t, :]                M=128, N=Ls,  K=128
// N = 128 matters: on B200 a 128x64x16 MMA takes about as long as a
// 128x128x16 one, so 64-token tiles spend twice the tensor time on QK^T.
// The tile is TMA-loaded once into 128B-swizzled shared memory, each 16 KB
// chunk holding one 64-column slice of both pages (rows 0-63 the first page,
// rows 64-127 the second), and it is the K-major B operand of QK^T and the
// MN-major B operand of PV.
//
// Operand placement (tensor memory holds 512 columns of 128 lanes):
//   tensor memory: O (Ls columns, fp32), S (128 columns, fp32) and the latent
//                  part of Q (Ls/2 columns, bf16 pairs) as the A operand of
//                  the first Ls/16 QK^T steps;
//   shared memory: the RoPE part of Q (A operand of the last R/16 QK^T steps)
//                  and P (A operand of PV), in the 128B-swizzled K-major layout.
//
// Precision: QK^T multiplies the bf16 inputs as they are.  PV multiplies the
// probabilities P, rounded to 16 bits, by the latent tile.  Rounding P to
// bf16 (8 significant bits) gives outputs with about 1.2e-3 relative RMS
// error on sequences of a few hundred tokens, falling to 3-7e-4 at 4K-32K
// tokens (the output's systematic part grows with length while the rounding
// noise averages out).  So the tiles of a sequence shorter than
// kExactPVBelow tokens run PV in fp16 (11 bits, about 1.5e-4): one MMA never
// mixes the two types, so after QK^T of such a tile has completed the softmax
// warps convert its latent rows in shared memory from bf16 to fp16 in place.
// A bf16 value is exactly an fp16 value only between 2^-14 and 65504, and the
// cache is the caller's (any transform, any norm weight), so each such tile
// first takes the maximum |value| of its valid rows across the softmax warps
// and scales the tile by a power of two (and P by its inverse) to bring that
// maximum into fp16's range, keeping bf16 only for tiles beyond that
// (pv_fp16_shift in attn_sm100_common.cuh).
// Longer sequences keep the bf16 tile and bf16 P, which costs no extra
// shared-memory traffic.  In both modes the rows past the end of the sequence
// are zeroed before PV reads the tile.
// All exponentials run on the special-function unit: moving a share of them
// to a polynomial on the FMA pipe measured slower here, since the softmax is
// bound by its latency chain, not by that unit's throughput.
//
// Warp roles (384 threads): warp 0 issues TMA loads into a ring of NST
// stages (page-table entries fetched a few pages ahead); warp 1 allocates
// tensor memory and issues the MMAs from one thread, polling for whichever
// of QK^T(next tile) and PV(oldest tile) is ready; warps 2-3 only complete
// the control warpgroup, whose registers go to the softmax; warps 4-11 are
// two softmax warpgroups.  Both own all 128 TMEM lanes (one head row per thread);
// warpgroup 0 takes score columns 0-63 of every tile, warpgroup 1 columns
// 64-127, and they agree on each row's running maximum through a per-tile
// exchange.  Each warpgroup rescales, and finally writes, its half of the O
// columns.  O is rescaled only when a row's running maximum grows by more
// than 8 (log2 units); a stale maximum only bounds p by 2^8.
//
// Every wait is bounded in time (SM clock cycles); a wait that runs out
// records TPLA_ERR_TIMEOUT in the device status word, sets a CTA-wide abort
// flag so all roles stop, and the kernel drains its TMA loads and MMAs
// before it frees tensor memory and returns.  No role waits on a plain CTA
// barrier while another may have stopped.
#include "tpla_internal.cuh"
#include "sm100_ptx.cuh"
#include "attn_sm100_common.cuh"

namespace tpla {
namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr int kSoftmaxWarp0 = 4;                // warps 4-11: two whole hardware warpgroups
// Register split.  Ten or twelve warps on four sub-partitions put three warps on some of them, which
// caps a thread at 168 registers, and the softmax path spills at that cap.  The control warpgroup
// (warps 0-3; the MMA issue code needs about 120) gives the rest of its share to the softmax
// warpgroups: launched at 168 per thread (64,512 registers), 4 warps x 120 + 8 warps x 192 per lane
// adds up to that total exactly, and neither side spills.
constexpr int kLaunchRegs = 168;
constexpr int kCtrlRegs = 120;
constexpr int kSoftmaxRegs = 192;
static_assert(32 * (4 * kCtrlRegs + 8 * kSoftmaxRegs) <= kLaunchRegs * kThreads, "register split");
constexpr int kSoftmaxWarps = 8;
constexpr float kRescaleThreshold = 8.0f;     // log2 units
constexpr int kExactPVBelow = 8192;           // sequences shorter than this run PV in fp16
constexpr int kPageAhead = 4;                 // page-table entries the producer loads ahead

template <int LS, int RD, int NST, int TT>
struct Cfg {
    static constexpr int kChunk = TT * 128;                    // TT rows x 128 bytes: a 64-column slice of the tile
    static constexpr int kHalf = kPage * 128;                  // one page's 64 rows of a chunk
    static constexpr int kChunksC = LS / 64;
    static constexpr int kStageBytes = (kChunksC + 1) * kChunk;   // latent chunks + the RoPE chunk
    static constexpr int kPChunk = 128 * 128;                  // P: 128 rows x 64 tokens x 2 B per chunk
    static constexpr int kPChunks = TT / 64;
    static constexpr int kEpiBytes = 32 * 1024 - kPChunks * kPChunk;   // epilogue staging beyond P (8 warps x 4 KB)
    static constexpr int kCvtShift = TT == 128 ? 10 : 9;       // log2 of the 16-byte pieces of one chunk
    static constexpr int kQpeBytes = 128 * 128;                // RoPE query: 128 rows x 64 x 2 B
    static constexpr int kColO = 0;
    static constexpr int kColS = LS;                           // 128 columns
    static constexpr int kColQ = LS + TT;                      // latent query, LS/2 columns
    static constexpr int kColsUsed = kColQ + LS / 2;
    static constexpr int kTmemCols = kColsUsed <= 128 ? 128 : (kColsUsed <= 256 ? 256 : 512);
    static constexpr int kStepsC = LS / 16;                    // QK^T steps over the latent
    static constexpr int kStepsR = RD / 16;                    // QK^T steps over the RoPE key
    static constexpr uint32_t kIdescQK = idesc_f16kind(128, TT, false, true);         // bf16 x bf16
    static constexpr uint32_t kIdescPVf16 = idesc_f16kind(128, LS, true, false);       // fp16 x fp16
    static constexpr uint32_t kIdescPVbf16 = idesc_f16kind(128, LS, true, true);       // bf16 x bf16
    static constexpr int kCvt = kChunksC * TT * 8 / (kSoftmaxWarps * 32);              // 16-byte pieces per thread
    static constexpr size_t kSmem = 1024 + (size_t)NST * kStageBytes + kPChunks * kPChunk + kEpiBytes + kQpeBytes;
    static_assert(kColsUsed <= 512, "tensor memory");
    static_assert(LS % 64 == 0 && RD == 64, "tile shape");
    static_assert(kCvt >= 1 && kChunksC * TT * 8 % (kSoftmaxWarps * 32) == 0, "conversion split");
    static_assert((TT == 64 || TT == 128) && (1 << kCvtShift) == TT * 8, "tile of one or two pages");
};

template <int NST>
struct Bars {
    uint64_t full[NST];
    uint64_t empty[NST];
    uint64_t s_full, s_free, p_full, o_done;
    uint64_t q_full, o_free, xmax, xsum, drain, never, vote;
    float xmax_buf[2][2][128];     // [tile parity][warpgroup][row]
    float xsum_buf[2][2][128];     // [segment parity][warpgroup][row]
    uint32_t vote_max[2][8];       // [tile parity][softmax warp]: largest |latent| bit pattern seen
    int pv_f16[2];                 // [tile parity]: PV of that tile runs in fp16
    uint32_t tmem_base;
    volatile int abort;
};

template <int LS, int RD, int NST, bool HALF, int TT>
__global__ void __launch_bounds__(kThreads, 1)
attn_sm100_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_o, Plan p,
                  const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ q_pe,
                  const int32_t* __restrict__ block_table, const int32_t* __restrict__ seq_lens, Workspace ws,
                  uint64_t wait_ns, int debug_stall) {
    using C = Cfg<LS, RD, NST, TT>;
    constexpr int kTileTok = TT;
    extern __shared__ uint8_t smem_raw[];
    // 1024-byte aligned base, by pointer arithmetic on the shared array so that every access
    // derived from it stays a shared-memory access
    uint8_t* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint8_t* p_smem = smem + NST * C::kStageBytes;          // P: one K chunk per 64 tokens (+ epilogue staging)
    uint8_t* qpe_smem = p_smem + C::kPChunks * C::kPChunk + C::kEpiBytes;   // RoPE query
    auto& bars = *reinterpret_cast<Bars<NST>*>(qpe_smem + C::kQpeBytes);
    const uint32_t stage0 = smem_addr(smem);
    const uint32_t p_addr = smem_addr(p_smem);
    const uint32_t qpe_addr = smem_addr(qpe_smem);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int w = blockIdx.x;

    // barriers first: this part touches no global memory and may overlap the previous kernel
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
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
        bars.abort = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
        prefetch_tensor_map(&tm_c);
        prefetch_tensor_map(&tm_k);
    }
    // every input may have been written by the previous kernel on the stream: wait for it
    pdl_wait();

    // every warp derives the same unit range from seq_lens
    const long long V = warp_total_weight(seq_lens, p);
    if (V == 0) return;
    const long long lo = warp_unit_at_weight(seq_lens, p, unit_lo(w, V, p.W));
    const long long hi = warp_unit_at_weight(seq_lens, p, unit_lo(w + 1, V, p.W));
    if (lo >= hi) {
        // a worker with no units leaves a zero-weight partial in its slot: the merge may count it
        // as a segment of the pair it falls inside
        for (int i = threadIdx.x; i < p.H; i += blockDim.x) ws.part_lse[(size_t)w * p.H + i] = -INFINITY;
        return;
    }
    const UnitPos pos0 = warp_locate_unit(seq_lens, p.B, p.max_pages, p.gc, lo);

    if (warp == 1) {
        tmem_alloc(smem_addr(&bars.tmem_base), C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bars.tmem_base;
    // 2 cycles per nanosecond bounds the clock from above (B200 runs at most 1.965 GHz)
    const Waiter wt{&bars.abort, p.status, wait_ns * 2};
    // Each role's code sits inside the branch that set its register budget, so that the compiler
    // allocates it within that budget.
    if (warp < kSoftmaxWarp0) {
        reg_dealloc<kCtrlRegs>();
        if (warp == 0) {
            // ------------------------------------------------------------ TMA producer
            if (lane == 0) {
                // Page-table entries are loaded kPageAhead units ahead of their TMA issue, as plain
                // loads that can all be in flight at once; an entry is checked when it is used.
                // (Prefetching the units a stage ring ahead into L2 measured slower on B200.)
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
                // every popped entry belongs to a unit of the range: an entry outside [0, num_pages)
                // is a caller error, recorded, and the page reads as zeros
                auto pop_page = [&]() -> int {
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
                    return page;
                };
                Tile t = make_tile(pos0, lo, lo, hi, kTileTok / kPage);
                long long j = 0;
                for (; t.u < hi; ++j) {
                    const int st = (int)(j % NST);
                    const uint32_t use = (uint32_t)(j / NST);
                    const int page0 = pop_page();
                    const int page1 = t.npages == 2 ? pop_page() : -1;
                    if (use > 0 && !wt.wait(smem_addr(&bars.empty[st]), (use - 1) & 1)) break;
                    const int shard = p.shard0 + t.pos.s;
                    if (t.begin && j > 0) {
                        // the softmax warps load this segment's query when the previous segment's last
                        // tile is done, a few tiles from now: have it in L2 by then
                        const __nv_bfloat16* qrow = q + (size_t)t.pos.b * p.H * p.L + (size_t)shard * LS;
                        for (int h = 0; h < p.H; ++h) prefetch_l2(qrow + (size_t)h * p.L, LS * 2);
                        prefetch_l2(q_pe + (size_t)t.pos.b * p.H * RD, (uint32_t)(p.H * RD * 2));
                    }
                    const uint32_t full = smem_addr(&bars.full[st]);
                    const uint32_t dst = stage0 + st * C::kStageBytes;
                    mbar_arrive_expect_tx(full, C::kStageBytes);
    #pragma unroll
                    for (int k = 0; k < kTileTok / kPage; ++k) {
                        // a missing or invalid page reads rows past the end of the tensor: TMA fills zeros
                        const int page = k == 0 ? page0 : page1;
                        const int yc = page >= 0 ? (page * p.g + shard) * kPage : p.num_pages * p.g * kPage;
                        const int yk = page >= 0 ? page * kPage : p.num_pages * kPage;
    #pragma unroll
                        for (int c = 0; c < C::kChunksC; ++c)
                            tma_load_2d(dst + c * C::kChunk + k * C::kHalf, &tm_c, full, c * 64, yc);
                        tma_load_2d(dst + C::kChunksC * C::kChunk + k * C::kHalf, &tm_k, full, 0, yk);
                    }
                    t = next_tile(t, seq_lens, p, lo, hi);
                }
                // All loads are issued: the next kernel (the combine) may launch once every CTA is
                // here.  Triggering at the start instead lets its CTAs pile onto the SMs whose workers
                // finish first, which unbalances the combine.
                pdl_trigger();
                // drain: the last use of every stage must have landed before the CTA exits
                for (long long x = j - NST < 0 ? 0 : j - NST; x < j; ++x) {
                    const int st = (int)(x % NST);
                    // bounded wait that ignores the abort flag (the copy is in flight either way)
                    const uint64_t t0 = globaltimer_ns();
                    while (!mbar_try_wait(smem_addr(&bars.full[st]), (uint32_t)(x / NST) & 1)) {
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
                // Issue whichever MMA is ready, polling without blocking: PV of the oldest tile as soon
                // as its P is in shared memory, QK^T of the next tile as soon as its stage has landed
                // and S has been read.  PV goes first when both are ready, since it releases a stage
                // for the next load.  (Issuing QK^T in several groups, to let a PV that becomes ready
                // meanwhile in sooner, measured much slower on B200: the issue of a group costs far
                // more than its MMAs.)  Each stream has its own tile cursor.
                Tile tq = make_tile(pos0, lo, lo, hi, kTileTok / kPage), tv = tq;
                long long jq = 0, jv = 0;
                int qseg = -1, vseg = -1;
                bool vbegun = false, vexact = false;
                long long idle_since = clock64();
                while (ok && tv.u < hi) {
                    bool did = false;
                    if (jv < jq) {
                        if (tv.begin && !vbegun) {
                            ++vseg;
                            vexact = tv.pos.T < kExactPVBelow;
                            vbegun = true;
                        }
                        if (mbar_test_wait(smem_addr(&bars.p_full), (uint32_t)(jv & 1)) &&
                            (!tv.begin || vseg == 0 ||
                             mbar_test_wait(smem_addr(&bars.o_free), (uint32_t)((vseg - 1) & 1)))) {
                            tc_fence_after();
                            const int st = (int)(jv % NST);
                            const uint32_t sb = stage0 + st * C::kStageBytes;
                            // a short segment's softmax warps chose this tile's PV type before they
                            // signalled P; a long segment's tiles are bf16
                            const uint32_t idesc_pv =
                                vexact && bars.pv_f16[jv & 1] ? C::kIdescPVf16 : C::kIdescPVbf16;
    #pragma unroll
                            for (int kk = 0; kk < kTileTok / 16; ++kk) {
                                // A: 16 tokens of P (K-major); B: the same 16 token rows of every latent chunk (MN-major)
                                const uint64_t ad = smem_desc_sw128(p_addr + (kk >> 2) * C::kPChunk + (kk & 3) * 32, 16, 1024);
                                const uint64_t bd = smem_desc_sw128(sb + kk * 2048, C::kChunk, 1024);
                                mma_ss(tmem + C::kColO, ad, bd, idesc_pv, (tv.begin && kk == 0) ? 0u : 1u);
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
                        const int st = (int)(jq % NST);
                        if ((!tq.begin || mbar_test_wait(smem_addr(&bars.q_full), (uint32_t)((qseg + 1) & 1))) &&
                            mbar_test_wait(smem_addr(&bars.full[st]), (uint32_t)((jq / NST) & 1)) &&
                            (jq == 0 || mbar_test_wait(smem_addr(&bars.s_free), (uint32_t)((jq - 1) & 1)))) {
                            if (tq.begin) ++qseg;
                            tc_fence_after();
                            const uint32_t sb = stage0 + st * C::kStageBytes;
                            const uint32_t d = tmem + C::kColS;
    #pragma unroll
                            for (int kk = 0; kk < C::kStepsC; ++kk) {
                                const uint64_t bd = smem_desc_sw128(sb + (kk >> 2) * C::kChunk + (kk & 3) * 32, 16, 1024);
                                mma_ts(d, tmem + C::kColQ + kk * 8, bd, C::kIdescQK, kk > 0 ? 1u : 0u);
                            }
    #pragma unroll
                            for (int kk = 0; kk < C::kStepsR; ++kk) {
                                const uint64_t ad = smem_desc_sw128(qpe_addr + kk * 32, 16, 1024);
                                const uint64_t bd = smem_desc_sw128(sb + C::kChunksC * C::kChunk + kk * 32, 16, 1024);
                                mma_ss(d, ad, bd, C::kIdescQK, 1u);
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
        }
    } else {
        reg_alloc<kSoftmaxRegs>();
        // ------------------------------------------------------------ softmax / epilogue (warps 4..11)
        const int sw = warp - kSoftmaxWarp0;              // 0..7
        const int wg = sw >> 2;                           // which half of the tile columns and of O
        const int quad = warp & 3;
        const int row = quad * 32 + lane;                 // TMEM lane (row of S, P, O and the query)
        const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
        // With at most 64 heads (HALF), lanes 64-127 carry the query of lanes 0-63, so their S rows
        // repeat rows 0-63 at no extra MMA cost, and all eight warps share the softmax: a head's
        // 128 score columns are split four ways (warpgroup x lower/upper lane half) instead of
        // two.  P rows 64-127 stay zero, so O rows 64-127 stay zero; only the lower half keeps O.
        const int hrow = HALF ? (row & 63) : row;         // head of this lane
        const bool upper = HALF && quad >= 2;
        const bool warp_active = (HALF ? (quad & 1) * 32 : quad * 32) < p.H;
        const bool row_active = hrow < p.H;
        const bool o_warp = warp_active && !upper;        // keeps, rescales and writes O rows
        const int tid_sm = threadIdx.x - kSoftmaxWarp0 * 32;   // 0..255
        // A negative scale is folded into the query: its bf16 sign bits are flipped on load (exact),
        // so the scores this kernel sees are multiplied by |scale| and the row maximum is the max.
        const float sc = fabsf(p.scale_log2);
        const uint32_t qflip = p.scale_log2 < 0.f ? 0x80008000u : 0u;
        constexpr int kOHalf = LS / 2;                    // O columns per warpgroup
        constexpr int kCols = HALF ? kTileTok / 4 : kTileTok / 2;   // score columns per thread
        const int cbase = wg * (kTileTok / 2) + (upper ? kCols : 0);  // the first of them
        long long last_o = -1;                            // highest PV index whose completion was observed
        int seg = -1;
        float m = -INFINITY, l = 0.f;                     // l: this thread's part of the row sum
        bool first_tile = true;
        bool exact = false;                               // segment short enough for fp16 PV tiles
        long long nvote = 0;                              // range votes taken (tiles of short segments)
        // PV(t) is the t-th completion of o_done; completions are in order, so observing PV(t)
        // covers all before it
        auto wait_o = [&](long long t) -> bool {
            if (t <= last_o) return true;
            if (!wt.wait(smem_addr(&bars.o_done), (uint32_t)(t & 1))) return false;
            last_o = t;
            tc_fence_after();
            return true;
        };
        // Query of one (b, shard) segment: the latent part into tensor memory as bf16 pairs (the
        // warpgroups take alternate 64-element chunks), the RoPE part into shared memory.  All
        // global loads are issued before the first store.  Called for the worker's first segment
        // here, and for each later one as soon as the previous segment's last S has been read
        // (its last QK^T, the final reader of both, has completed), ahead of that segment's
        // epilogue, so that the next QK^T overlaps it.
        auto load_q = [&](const UnitPos& qp) {
            constexpr int kQc = (C::kChunksC + 1) / 2;    // latent chunks per warpgroup
            const int shard = p.shard0 + qp.s;
            if (warp_active) {
                const uint4* qs = reinterpret_cast<const uint4*>(q + ((size_t)qp.b * p.H + hrow) * p.L +
                                                                 (size_t)shard * LS);
                const uint4* qpp = reinterpret_cast<const uint4*>(q_pe + ((size_t)qp.b * p.H + hrow) * RD);
                uint4 x[kQc][8], xp[4];
#pragma unroll
                for (int i = 0; i < kQc; ++i) {
                    const int c = wg + 2 * i;
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        x[i][v] = (row_active && c < C::kChunksC) ? __ldg(qs + c * 8 + v) : make_uint4(0, 0, 0, 0);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) xp[k] = row_active ? __ldg(qpp + wg * 4 + k) : make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < kQc; ++i) {
                    const int c = wg + 2 * i;
                    if (c < C::kChunksC) {
                        uint32_t r[32];
#pragma unroll
                        for (int v = 0; v < 8; ++v) {
                            r[4 * v + 0] = x[i][v].x ^ qflip; r[4 * v + 1] = x[i][v].y ^ qflip;
                            r[4 * v + 2] = x[i][v].z ^ qflip; r[4 * v + 3] = x[i][v].w ^ qflip;
                        }
                        tmem_st32(lane_base + C::kColQ + c * 32, r);
                    }
                }
                tmem_wait_st();
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    *reinterpret_cast<uint4*>(qpe_smem + sw128_offset(row, wg * 4 + k)) =
                        make_uint4(xp[k].x ^ qflip, xp[k].y ^ qflip, xp[k].z ^ qflip, xp[k].w ^ qflip);
            } else {
                // rows past H: zero RoPE query (the latent columns of these lanes are never read)
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    *reinterpret_cast<uint4*>(qpe_smem + sw128_offset(row, wg * 4 + k)) = make_uint4(0, 0, 0, 0);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            warp_arrive(smem_addr(&bars.q_full));
        };
        if (HALF && upper) {
            // P rows 64-127 (this warp's lanes, in every K chunk) stay zero
#pragma unroll
            for (int c = 0; c < C::kPChunks; ++c)
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    *reinterpret_cast<uint4*>(p_smem + c * C::kPChunk + sw128_offset(row, k)) = make_uint4(0, 0, 0, 0);
        }
        Tile t = make_tile(pos0, lo, lo, hi, kTileTok / kPage);
        load_q(pos0);
        long long j = 0;
        for (; t.u < hi; ++j) {
            const UnitPos pos = t.pos;
            if (t.begin) {
                ++seg;
                if (wg == 0 && lane == 0) (void)effective_len(seq_lens, pos.b, p.max_pages, p.status);
                m = -INFINITY;
                l = 0.f;
                first_tile = true;
                exact = pos.T < kExactPVBelow;
            }
            // tokens of this tile that belong to the sequence (rows 0-63 the first page, 64-127 the second)
            const int loaded = t.npages * kPage;
            const int valid = min(loaded, pos.T - pos.tile * kPage);
            const bool tail = valid < kTileTok;
            if (!wt.wait(smem_addr(&bars.s_full), (uint32_t)(j & 1))) break;
            tc_fence_after();
            float s[kCols];
            if (warp_active) {
                if constexpr (kCols == 16) {
                    uint32_t r[16];
                    tmem_ld16(lane_base + C::kColS + cbase, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int k = 0; k < 16; ++k) s[k] = __uint_as_float(r[k]);
                } else {
#pragma unroll
                    for (int h = 0; h < kCols / 32; ++h) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + C::kColS + cbase + 32 * h, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) s[32 * h + k] = __uint_as_float(r[k]);
                    }
                }
            } else {
#pragma unroll
                for (int k = 0; k < kCols; ++k) s[k] = 0.f;
            }
            tc_fence_before();
            warp_arrive(smem_addr(&bars.s_free));
            uint8_t* sb = smem + (int)(j % NST) * C::kStageBytes;

            // row maximum of the raw scores over this warpgroup's valid columns
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
            // Reference maximum of this tile's exponentials, decided without waiting for the other
            // warpgroup: the running maximum m, raised to this warpgroup's own maximum when that
            // exceeds m by more than the threshold (always on a segment's first tile).  The raised
            // references are exchanged after P is formed; the row's new running maximum is the
            // largest of m and them, and a warpgroup whose reference is below it scales its P down.
            const float m_loc = ext * sc;                                   // -inf: no valid column
            const bool raise = warp_active && m_loc > -INFINITY && (first_tile || m_loc > m + kRescaleThreshold);
            const float m_ref = raise ? m_loc : (m > -INFINITY ? m : 0.f);  // 0: no valid column yet, P = 0
            bars.xmax_buf[j & 1][wg][row] = raise ? m_loc : -INFINITY;
            warp_arrive(smem_addr(&bars.xmax));
            // PV type of this tile (pv_fp16_shift): a tile of a short segment, where the rounding of
            // P would dominate the error, runs PV in fp16 with the latent values scaled by 2^e and P
            // by 2^-e; from kExactPVBelow tokens on, and for tiles whose largest |value| is outside
            // fp16's reach even when scaled, it keeps bf16.  The softmax warps agree on the tile's
            // largest |value| through the vote barrier: each posts the largest bit pattern of |value|
            // over its share of the tile's valid rows.
            bool f16 = false;
            float cshift = 1.f, pshift = 1.f;             // 2^e for the latent tile, 2^-e for P
            if (exact) {
                // all of this thread's loads in flight at once; rows past the sequence end are
                // loaded (they lie inside the stage) but not counted
                uint32_t mx = 0;
                uint4 vt[C::kCvt];
#pragma unroll
                for (int k = 0; k < C::kCvt; ++k) {
                    const int i = tid_sm + k * kSoftmaxWarps * 32;
                    const int rr = (i >> 3) & (kTileTok - 1);
                    vt[k] = *reinterpret_cast<const uint4*>(sb + (i >> C::kCvtShift) * C::kChunk + rr * 128 + (i & 7) * 16);
                }
#pragma unroll
                for (int k = 0; k < C::kCvt; ++k) {
                    const int rr = ((tid_sm + k * kSoftmaxWarps * 32) >> 3) & (kTileTok - 1);
                    if (rr < valid)
                        mx = __vmaxu2(mx, __vmaxu2(__vmaxu2(vt[k].x & 0x7FFF7FFFu, vt[k].y & 0x7FFF7FFFu),
                                                  __vmaxu2(vt[k].z & 0x7FFF7FFFu, vt[k].w & 0x7FFF7FFFu)));
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
                // a long segment's tiles are bf16 without a vote: pack here, beside the exponentials
                if (!exact) pack();
            } else {
#pragma unroll
                for (int k = 0; k < kCols / 2; ++k) pk[k] = 0u;
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
                if (warp_active) pack();
            }
            if (f16) {
                // this tile's latent rows -> fp16 (rows past the sequence end -> 0) for PV;
                // QK^T has finished reading them.  The 128B swizzle only permutes the 16-byte
                // pieces within a row, so row rr is the 128 bytes at rr * 128 of its chunk.
#pragma unroll 4
                for (int k = 0; k < C::kCvt; ++k) {
                    const int i = tid_sm + k * kSoftmaxWarps * 32;
                    const int rr = (i >> 3) & (kTileTok - 1);
                    uint4* ptr = reinterpret_cast<uint4*>(sb + (i >> C::kCvtShift) * C::kChunk + rr * 128 + (i & 7) * 16);
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
            } else if (valid < loaded) {
                // bf16 tile kept as it is; only the loaded rows past the sequence end are zeroed
                // (the rows of a page that was not loaded are zero already)
                const int rows = loaded - valid;
                for (int i = tid_sm; i < C::kChunksC * rows * 8; i += kSoftmaxWarps * 32) {
                    const int c = i / (rows * 8), rr = valid + (i / 8) % rows, seg16 = i % 8;
                    *reinterpret_cast<uint4*>(sb + c * C::kChunk + rr * 128 + seg16 * 16) = make_uint4(0, 0, 0, 0);
                }
            }
            // the other warpgroup's raised reference, the row's new running maximum, and the rescales
            if (!wt.wait(smem_addr(&bars.xmax), (uint32_t)(j & 1))) break;
            {
                float other = bars.xmax_buf[j & 1][wg ^ 1][row];
                if (HALF)
                    other = fmaxf(other, fmaxf(bars.xmax_buf[j & 1][wg][row ^ 64], bars.xmax_buf[j & 1][wg ^ 1][row ^ 64]));
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
                        // (an upper-half warp only rescales its part of l)
                        const float alpha = m_new > m ? ex2_approx(m - m_new) : 1.0f;
                        if (o_warp && !wait_o(j - 1)) alive = false;
                        if (!o_warp) {
                            l *= alpha;
                        } else if (alive) {
#pragma unroll 1
                            for (int c = 0; c < kOHalf / 32; ++c) {
                                const uint32_t ta = lane_base + C::kColO + wg * kOHalf + c * 32;
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
            {
                // this thread's columns are the 16-byte pieces from (cbase mod 64) / 8 on, in its
                // head's row of K chunk cbase / 64 of P (64 tokens per chunk)
                uint8_t* pb = p_smem + (cbase >> 6) * C::kPChunk;
                const int k0 = (cbase & 63) >> 3;
#pragma unroll
                for (int k = 0; k < kCols / 8; ++k)
                    *reinterpret_cast<uint4*>(pb + sw128_offset(hrow, k0 + k)) =
                        make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
            }
            if (exact && tid_sm == 0) bars.pv_f16[j & 1] = f16 ? 1 : 0;   // read by the issuer after p_full
            fence_proxy_async_smem();
            warp_arrive(smem_addr(&bars.p_full));
            first_tile = false;

            const Tile tn = next_tile(t, seq_lens, p, lo, hi);
            if (t.end) {
                if (tn.u < hi) load_q(tn.pos);
                if (!wait_o(j)) break;
                // the two warpgroups' halves of the softmax sum
                bars.xsum_buf[seg & 1][wg][row] = l;
                warp_arrive(smem_addr(&bars.xsum));
                if (!wt.wait(smem_addr(&bars.xsum), (uint32_t)(seg & 1))) break;
                float lt = l + bars.xsum_buf[seg & 1][wg ^ 1][row];
                if (HALF) lt += bars.xsum_buf[seg & 1][wg][row ^ 64] + bars.xsum_buf[seg & 1][wg ^ 1][row ^ 64];
                const long long u_first = t.u - pos.tile;       // unit of page 0 of this (b, s)
                const int slot = u_first >= lo ? p.W + pos.b * p.gc + pos.s : w;
                if (o_warp) {
                    // The normalised rows go out 32 columns at a time: staged in this warp's own
                    // rows of the P buffer (free: the segment's last PV has completed), 128B-swizzled,
                    // and written by a TMA store of a 32 x 32 box.  Rows past H lie outside the
                    // tensor map and are not written.  Each box waits until the previous store has
                    // read the buffer; the last wait comes before P is written again.
                    const float inv_l = 1.0f / lt;
                    uint8_t* stile = p_smem + (wg * 4 + quad) * 4096;   // P and the staging beyond it
#pragma unroll 1
                    for (int c = 0; c < kOHalf / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld32(lane_base + C::kColO + wg * kOHalf + c * 32, r);
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
                            tma_store_3d(&tm_o, smem_addr(stile), wg * kOHalf + c * 32, quad * 32, slot);
                            bulk_commit();
                        }
                    }
                    if (lane == 0) bulk_wait_read_all();
                    __syncwarp();
                    if (row_active && wg == 0) ws.part_lse[(size_t)slot * p.H + row] = m + log2f(lt);
                }
                tc_fence_before();
                warp_arrive(smem_addr(&bars.o_free));
            }
            t = tn;
        }
    }

    // the partial outputs' TMA stores have completed when the CTA exits
    if (warp >= kSoftmaxWarp0 && lane == 0) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

template <int LS, int RD, int NST, bool HALF, int TT>
cudaError_t launch_t(const Plan& p, const __nv_bfloat16* q, const __nv_bfloat16* q_pe, const __nv_bfloat16* ckv,
                     const __nv_bfloat16* kpe, const int32_t* bt, const int32_t* seq_lens, Workspace ws,
                     uint64_t wait_ns, int debug_stall, cudaStream_t stream) {
    using C = Cfg<LS, RD, NST, TT>;
    CUtensorMap tc, tk;
    if (!make_map(&tc, ckv, LS, (uint64_t)p.num_pages * p.g * kPage)) return cudaErrorInvalidValue;
    if (!make_map(&tk, kpe, RD, (uint64_t)p.num_pages * kPage)) return cudaErrorInvalidValue;
    CUtensorMap to;
    if (!make_map_o(&to, ws.part_o, LS, p.H, (uint64_t)num_slots(p))) return cudaErrorInvalidValue;
    const size_t smem = C::kSmem + sizeof(Bars<NST>);
    static_assert(C::kTmemCols < 512 || C::kSmem > 116 * 1024, "a 512-column TMEM allocation needs one CTA per SM");
    static_assert(C::kSmem + sizeof(Bars<NST>) <= 227 * 1024, "shared memory");
    auto kern = attn_sm100_kernel<LS, RD, NST, HALF, TT>;
    static unsigned long long attr_done = 0;
    cudaError_t e = set_smem_once(kern, smem, &attr_done);
    if (e != cudaSuccess) return e;
    // The register split draws on the registers the CTA is launched with: a build that gives the
    // kernel fewer than kLaunchRegs per thread would leave the softmax warps waiting for registers
    // that never come, so it is refused here.
    static int regs_ok = -1;
    if (regs_ok < 0) {
        cudaFuncAttributes fa;
        e = cudaFuncGetAttributes(&fa, kern);
        if (e != cudaSuccess) return e;
        regs_ok = fa.numRegs >= kLaunchRegs ? 1 : 0;
    }
    if (!regs_ok) return cudaErrorNotSupported;
    return launch_pdl(kern, dim3(p.W), dim3(kThreads), smem, stream, tc, tk, to, p, q, q_pe, bt, seq_lens, ws,
                      wait_ns, debug_stall);
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
    const bool half = p.H <= 64;
    // stages: as many as fit beside P, the epilogue staging and the RoPE query (two-page tiles: the
    // 128-token tile of L/g = 256 takes 80 KB; one-page tiles: 40 KB)
#define TPLA_LAUNCH(LS, NST, TT)                                                                                   \
    return half ? launch_t<LS, 64, NST, true, TT>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, wait_ns,         \
                                                  debug_stall, stream)                                             \
                : launch_t<LS, 64, NST, false, TT>(p, q, q_pe, ckv, kpe, block_table, seq_lens, ws, wait_ns,        \
                                                   debug_stall, stream)
    if (p.tile_tok == 64) {
        switch (p.Ls) {
            case 256: TPLA_LAUNCH(256, 4, 64);
            case 128: TPLA_LAUNCH(128, 7, 64);
            case 64: TPLA_LAUNCH(64, 10, 64);
        }
    } else {
        switch (p.Ls) {
            case 256: TPLA_LAUNCH(256, 2, 128);
            case 128: TPLA_LAUNCH(128, 3, 128);
            case 64: TPLA_LAUNCH(64, 5, 128);
        }
    }
#undef TPLA_LAUNCH
    return cudaErrorNotSupported;
}

}  // namespace tpla
