// Host side of the C ABI declared in include/tpla.h: argument validation,
// the split-KV plan, workspace carving, kernel dispatch and the device
// status word.  Every check that can be made without the GPU runs before any
// CUDA call, so a bad argument returns its status with nothing enqueued.
#include "tpla_internal.cuh"

#include <cmath>
#include <cstdio>
#include <mutex>

namespace tpla {

// Per-device status word (bits kStatusIndex, kStatusTimeout), set by kernels.
__device__ unsigned int g_device_status;

namespace {

int g_opt_kernel = 0;        // TPLA_OPT_ATTENTION_KERNEL
int g_opt_max_workers = 0;   // TPLA_OPT_MAX_WORKERS
int g_opt_wait_limit = 0;    // TPLA_OPT_WAIT_LIMIT
int g_opt_debug_stall = 0;   // TPLA_OPT_DEBUG_STALL
int g_opt_tile_tokens = 0;   // TPLA_OPT_TILE_TOKENS
int g_last_kernel = 0;       // TPLA_OPT_LAST_ATTENTION_KERNEL

// Fewest units a tcgen05 worker gets: keeps the partial traffic small at batch 1.  The CUDA-core
// kernel is bound by arithmetic, not by that traffic, and spreads the units as widely as it can.
constexpr int kMinUnitsPerWorker = 4;
// A worker whose range ends one (sequence, shard) and starts the next stops its stream for the
// first one's epilogue and the second one's query load: measured on B200 at about as long as
// this many units of streaming.
constexpr long long kSwitchUnits = 8;
// Tokens per tile of the tcgen05 kernel for L/g <= 256 (TPLA_OPT_TILE_TOKENS = 0).
constexpr int kDefaultTileTokens = 128;

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
unsigned* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int check_dims(const tpla_dims_t* d) {
    if (!d) return TPLA_ERR_INVALID_ARG;
    if (d->B < 0 || d->H <= 0 || d->L <= 0 || d->R <= 0 || d->dv <= 0 || d->g <= 0 ||
        d->max_pages_per_seq <= 0 || d->num_pages <= 0)
        return TPLA_ERR_INVALID_ARG;
    if (!std::isfinite(d->softmax_scale)) return TPLA_ERR_INVALID_ARG;
    if (d->page_size != kPage) return TPLA_ERR_UNSUPPORTED;
    if (d->H > 128) return TPLA_ERR_UNSUPPORTED;
    if (!(d->g == 1 || d->g == 2 || d->g == 4 || d->g == 8)) return TPLA_ERR_UNSUPPORTED;
    if (!pow2(d->L) || d->L < 64 || d->L > 1024) return TPLA_ERR_UNSUPPORTED;
    if (d->L % d->g) return TPLA_ERR_UNSUPPORTED;
    const int Ls = d->L / d->g;
    if (Ls < 32 || Ls > 512) return TPLA_ERR_UNSUPPORTED;
    if (!(d->R == 16 || d->R == 32 || d->R == 64)) return TPLA_ERR_UNSUPPORTED;
    if (d->dv % 8 || d->dv > 256) return TPLA_ERR_UNSUPPORTED;
    if ((long long)d->max_pages_per_seq * kPage > (1ll << 30)) return TPLA_ERR_UNSUPPORTED;
    return TPLA_OK;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

size_t ws_lse_bytes(const tpla_dims_t* d) {
    return align_up((size_t)(kMaxWorkers + (size_t)d->B * d->g) * d->H * sizeof(float), 256);
}

// Workspace: 256-byte header | log-sum-exps [kMaxWorkers + B*g][H] | partial outputs [slots][H][L/g].
// `slots` is kMaxWorkers + B*g for a caller's workspace.
size_t ws_part_bytes(const tpla_dims_t* d, size_t slots) {
    return align_up(slots * d->H * (size_t)(d->L / d->g) * sizeof(float), 256);
}

size_t ws_bytes_for(const tpla_dims_t* d) {
    const size_t slots = (size_t)kMaxWorkers + (size_t)d->B * d->g;
    return 256 + ws_lse_bytes(d) + ws_part_bytes(d, slots);
}

int device_info(unsigned** status, int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TPLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TPLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (!g_status_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_device_status) != cudaSuccess) return TPLA_ERR_CUDA;
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TPLA_ERR_CUDA;
        g_sm_count[dev] = n;
        g_status_ptr[dev] = static_cast<unsigned*>(ptr);
    }
    if (status) *status = g_status_ptr[dev];
    if (sms) *sms = g_sm_count[dev];
    return TPLA_OK;
}

// Validation common to the decode stages.  shard == -1: all shards.
int check_decode(const tpla_dims_t* d, int shard, const void* q, const void* q_pe, const void* ckv,
                 const void* kpe, const int32_t* block_table, const int32_t* seq_lens,
                 void* workspace, size_t ws_bytes) {
    int st = check_dims(d);
    if (st) return st;
    if (shard < -1 || shard >= d->g) return TPLA_ERR_INVALID_ARG;
    if (d->B == 0) return TPLA_OK;
    if (!q || !q_pe || !ckv || !kpe || !seq_lens) return TPLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(q_pe) || !aligned16(ckv) || !aligned16(kpe) || !aligned16(seq_lens))
        return TPLA_ERR_INVALID_ARG;
    if (block_table && !aligned16(block_table)) return TPLA_ERR_INVALID_ARG;
    if (!block_table && (long long)d->B * d->max_pages_per_seq > d->num_pages) return TPLA_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return TPLA_ERR_WORKSPACE;
    if (ws_bytes < ws_bytes_for(d)) return TPLA_ERR_WORKSPACE;
    return TPLA_OK;
}

int make_plan(const tpla_dims_t* d, int shard, Plan* p) {
    unsigned* status = nullptr;
    int sms = 0;
    int st = device_info(&status, &sms);
    if (st) return st;
    p->B = d->B; p->H = d->H; p->L = d->L; p->R = d->R; p->dv = d->dv; p->g = d->g;
    p->Ls = d->L / d->g;
    p->gc = shard < 0 ? d->g : 1;
    p->shard0 = shard < 0 ? 0 : shard;
    p->max_pages = d->max_pages_per_seq;
    p->num_pages = d->num_pages;
    p->scale_log2 = d->softmax_scale * kLog2e;
    p->status = status;
    // the attention kernel: tcgen05 where the shape has a variant (unless the CUDA-core kernel is
    // forced), else the CUDA-core kernel; a forced tcgen05 kernel without a variant is an error
    const bool tc = sm100_supports(*p), wide = sm100_wide_supports(*p);
    if (g_opt_kernel == 2 && !tc && !wide) return TPLA_ERR_UNSUPPORTED;
    p->kernel = g_opt_kernel == 1 ? kKernelSimt : (tc ? kKernelSm100 : (wide ? kKernelSm100Wide : kKernelSimt));
    p->tile_tok = g_opt_tile_tokens ? g_opt_tile_tokens : kDefaultTileTokens;
    // split-KV cost weights: a tile of a sequence shorter than 8192 tokens takes the tcgen05
    // kernels' fp16 PV path (a range vote and an in-place conversion of the tile), measured at
    // about 1.3x the cost of a long sequence's tile; the CUDA-core kernel has one cost
    const bool tc_kernel = p->kernel == kKernelSm100 || p->kernel == kKernelSm100Wide;
    p->w_long = tc_kernel ? 3 : 1;
    p->w_short = tc_kernel ? 4 : 1;
    p->short_below = tc_kernel ? 8192 : 0;
    // workers: one per SM (a CTA pair per worker for the wide kernel), at most kMaxWorkers
    int cap = p->kernel == kKernelSm100Wide ? sms / 2 : sms;
    cap = cap < kMaxWorkers ? cap : kMaxWorkers;
    if (g_opt_max_workers > 0 && g_opt_max_workers < cap) cap = g_opt_max_workers;
    const long long umax = (long long)p->gc * d->B * d->max_pages_per_seq;
    const int min_units = p->kernel == kKernelSm100 ? kMinUnitsPerWorker : 1;
    long long w = (umax + min_units - 1) / min_units;
    w = w < 1 ? 1 : (w > cap ? cap : w);
    // With a multiple of the (sequence, shard) pair count as the worker count, equal-length pairs
    // split at worker boundaries and no worker switches pairs.  Take it when, for pairs of the
    // longest length, the longer ranges cost less than one switch.
    const long long pairs = (long long)p->gc * d->B, n = d->max_pages_per_seq;
    if (pairs > 1 && pairs <= w) {
        const long long wa = (w / pairs) * pairs;
        if (pairs * n * w <= (pairs * n + kSwitchUnits * w) * wa) w = wa;
    }
    p->W = (int)w;
    return TPLA_OK;
}

// Workspace: 256-byte header | log-sum-exps | partial outputs.  The log-sum-exp block is sized for
// kMaxWorkers + B*g slots in every path (ws_lse_bytes), so the partial outputs start at the same
// offset whatever worker count a call uses; the partial region needs (W + B*g) slots of H*(L/g)
// floats, which the caller's workspace (sized for kMaxWorkers) and the static scratch (W clamped
// to fit) both provide.
Workspace carve(void* workspace, const tpla_dims_t* d) {
    char* base = static_cast<char*>(workspace) + 256;
    Workspace w;
    w.part_lse = reinterpret_cast<float*>(base);
    w.part_o = reinterpret_cast<float*>(base + ws_lse_bytes(d));
    return w;
}

// The attention pass of plan p, on the kernel the plan chose; records which one was launched.
int launch_attention(const Plan& p, const tpla_bf16* q, const tpla_bf16* q_pe, const tpla_bf16* ckv,
                     const tpla_bf16* kpe, const int32_t* block_table, const int32_t* seq_lens, Workspace w,
                     cudaStream_t s) {
    auto bq = reinterpret_cast<const __nv_bfloat16*>(q);
    auto bqp = reinterpret_cast<const __nv_bfloat16*>(q_pe);
    auto bc = reinterpret_cast<const __nv_bfloat16*>(ckv);
    auto bk = reinterpret_cast<const __nv_bfloat16*>(kpe);
    cudaError_t e;
    switch (p.kernel) {
        case kKernelSm100:
            e = launch_attention_sm100(p, bq, bqp, bc, bk, block_table, seq_lens, w, g_opt_wait_limit,
                                       g_opt_debug_stall, s);
            break;
        case kKernelSm100Wide:
            e = launch_attention_sm100_wide(p, bq, bqp, bc, bk, block_table, seq_lens, w, g_opt_wait_limit,
                                            g_opt_debug_stall, s);
            break;
        default:
            e = launch_attention_simt(p, bq, bqp, bc, bk, block_table, seq_lens, w, s);
            break;
    }
    g_last_kernel = p.kernel;
    if (e == cudaErrorNotSupported) return TPLA_ERR_UNSUPPORTED;
    return e == cudaSuccess ? TPLA_OK : TPLA_ERR_CUDA;
}

int run_attention(const tpla_dims_t* d, int shard, const tpla_bf16* q, const tpla_bf16* q_pe,
                  const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
                  const int32_t* seq_lens, void* workspace, size_t ws_bytes, void* stream) {
    int st = check_decode(d, shard, q, q_pe, ckv, kpe, block_table, seq_lens, workspace, ws_bytes);
    if (st || d->B == 0) return st;
    Plan p;
    if ((st = make_plan(d, shard, &p))) return st;
    return launch_attention(p, q, q_pe, ckv, kpe, block_table, seq_lens, carve(workspace, d),
                            static_cast<cudaStream_t>(stream));
}

int run_combine(const tpla_dims_t* d, int shard, const int32_t* seq_lens, const tpla_bf16* w_uv,
                float* out, void* workspace, size_t ws_bytes, void* stream) {
    int st = check_dims(d);
    if (st) return st;
    if (shard < -1 || shard >= d->g) return TPLA_ERR_INVALID_ARG;
    if (d->B == 0) return TPLA_OK;
    if (!seq_lens || !out || !aligned16(out)) return TPLA_ERR_INVALID_ARG;
    if (w_uv && !aligned16(w_uv)) return TPLA_ERR_INVALID_ARG;
    if (!workspace || !aligned16(workspace)) return TPLA_ERR_WORKSPACE;
    if (ws_bytes < ws_bytes_for(d)) return TPLA_ERR_WORKSPACE;
    Plan p;
    if ((st = make_plan(d, shard, &p))) return st;
    cudaError_t e = launch_combine(p, seq_lens, reinterpret_cast<const __nv_bfloat16*>(w_uv), out,
                                   carve(workspace, d), static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? TPLA_OK : TPLA_ERR_CUDA;
}

int run_decode(const tpla_dims_t* d, int shard, const tpla_bf16* q, const tpla_bf16* q_pe,
               const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
               const int32_t* seq_lens, const tpla_bf16* w_uv, float* out, void* workspace,
               size_t ws_bytes, void* stream) {
    int st = check_decode(d, shard, q, q_pe, ckv, kpe, block_table, seq_lens, workspace, ws_bytes);
    if (st) return st;
    if (d->B > 0 && (!out || !aligned16(out))) return TPLA_ERR_INVALID_ARG;
    if (w_uv && !aligned16(w_uv)) return TPLA_ERR_INVALID_ARG;
    if ((st = run_attention(d, shard, q, q_pe, ckv, kpe, block_table, seq_lens, workspace, ws_bytes, stream)))
        return st;
    return run_combine(d, shard, seq_lens, w_uv, out, workspace, ws_bytes, stream);
}

// Cache append of every shard (shard == -1) into the g-shard cache, or of shard `shard` alone into a
// one-shard cache (one tensor-parallel rank's).
int run_append(const tpla_dims_t* dims, int shard, const tpla_bf16* latent_raw, const tpla_bf16* kpe_new,
               int transform, const float* R_dense, const float* norm_weight, float eps, const int32_t* positions,
               const int32_t* block_table, tpla_bf16* ckv_cache, tpla_bf16* kpe_cache, void* stream) {
    int st = check_dims(dims);
    if (st) return st;
    if (transform < TPLA_TRANSFORM_NONE || transform > TPLA_TRANSFORM_BLOCK_HADAMARD) return TPLA_ERR_INVALID_ARG;
    if (!(eps >= 0.f) || !std::isfinite(eps)) return TPLA_ERR_INVALID_ARG;
    if (dims->B == 0) return TPLA_OK;
    if (!latent_raw || !kpe_new || !positions || !ckv_cache || !kpe_cache) return TPLA_ERR_INVALID_ARG;
    if (transform == TPLA_TRANSFORM_DENSE && !R_dense) return TPLA_ERR_INVALID_ARG;
    if (!aligned16(ckv_cache) || !aligned16(kpe_cache) || !aligned16(latent_raw) || !aligned16(kpe_new))
        return TPLA_ERR_INVALID_ARG;
    if (!block_table && (long long)dims->B * dims->max_pages_per_seq > dims->num_pages)
        return TPLA_ERR_INVALID_ARG;
    unsigned* status = nullptr;
    if ((st = device_info(&status, nullptr))) return st;
    cudaError_t e = launch_append(*dims, shard, reinterpret_cast<const __nv_bfloat16*>(latent_raw),
                                  reinterpret_cast<const __nv_bfloat16*>(kpe_new), transform, R_dense,
                                  norm_weight, eps, positions, block_table,
                                  reinterpret_cast<__nv_bfloat16*>(ckv_cache),
                                  reinterpret_cast<__nv_bfloat16*>(kpe_cache), status,
                                  static_cast<cudaStream_t>(stream));
    if (e == cudaErrorNotSupported) return TPLA_ERR_UNSUPPORTED;
    return e == cudaSuccess ? TPLA_OK : TPLA_ERR_CUDA;
}

}  // namespace
}  // namespace tpla

using namespace tpla;

extern "C" {

const char* tpla_status_string(int status) {
    switch (status) {
        case TPLA_OK: return "TPLA_OK";
        case TPLA_ERR_INVALID_ARG: return "TPLA_ERR_INVALID_ARG: null, negative or misaligned argument";
        case TPLA_ERR_UNSUPPORTED: return "TPLA_ERR_UNSUPPORTED: size outside the supported set";
        case TPLA_ERR_LAYOUT: return "TPLA_ERR_LAYOUT: cache layout does not match the call";
        case TPLA_ERR_WORKSPACE: return "TPLA_ERR_WORKSPACE: workspace missing or too small";
        case TPLA_ERR_CUDA: return "TPLA_ERR_CUDA: CUDA runtime error";
        case TPLA_ERR_TIMEOUT: return "TPLA_ERR_TIMEOUT: a bounded device wait ran out";
        case TPLA_ERR_INDEX: return "TPLA_ERR_INDEX: device-side index out of range";
    }
    return "unknown tpla status";
}

size_t tpla_decode_workspace_size(const tpla_dims_t* dims) {
    if (check_dims(dims)) return 0;
    return ws_bytes_for(dims);
}

int tpla_decode(const tpla_dims_t* dims, const tpla_bf16* q, const tpla_bf16* q_pe,
                const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
                const int32_t* seq_lens, const tpla_bf16* w_uv, float* out, void* workspace,
                size_t ws_bytes, void* stream) {
    return run_decode(dims, -1, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace, ws_bytes,
                      stream);
}

int tpla_decode_shard(const tpla_dims_t* dims, int shard, const tpla_bf16* q, const tpla_bf16* q_pe,
                      const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
                      const int32_t* seq_lens, const tpla_bf16* w_uv, float* out, void* workspace,
                      size_t ws_bytes, void* stream) {
    if (dims && (shard < 0 || shard >= dims->g)) return TPLA_ERR_INVALID_ARG;
    return run_decode(dims, shard, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace,
                      ws_bytes, stream);
}

int mla_decode(const tpla_dims_t* dims, const tpla_bf16* q, const tpla_bf16* q_pe,
               const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
               const int32_t* seq_lens, const tpla_bf16* w_uv, float* out, void* workspace,
               size_t ws_bytes, void* stream) {
    if (!dims) return TPLA_ERR_INVALID_ARG;
    if (dims->g != 1) return TPLA_ERR_LAYOUT;
    return run_decode(dims, -1, q, q_pe, ckv, kpe, block_table, seq_lens, w_uv, out, workspace, ws_bytes,
                      stream);
}

int tpla_attention(const tpla_dims_t* dims, int shard, const tpla_bf16* q, const tpla_bf16* q_pe,
                   const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
                   const int32_t* seq_lens, void* workspace, size_t ws_bytes, void* stream) {
    return run_attention(dims, shard, q, q_pe, ckv, kpe, block_table, seq_lens, workspace, ws_bytes, stream);
}

int tpla_combine(const tpla_dims_t* dims, int shard, const int32_t* seq_lens, const tpla_bf16* w_uv,
                 float* out, void* workspace, size_t ws_bytes, void* stream) {
    return run_combine(dims, shard, seq_lens, w_uv, out, workspace, ws_bytes, stream);
}

int tpla_append_kv(const tpla_dims_t* dims, const tpla_bf16* latent_raw, const tpla_bf16* kpe_new,
                   int transform, const float* R_dense, const float* norm_weight, float eps,
                   const int32_t* positions, const int32_t* block_table, tpla_bf16* ckv_cache,
                   tpla_bf16* kpe_cache, void* stream) {
    return run_append(dims, -1, latent_raw, kpe_new, transform, R_dense, norm_weight, eps, positions, block_table,
                      ckv_cache, kpe_cache, stream);
}

int tpla_append_kv_shard(const tpla_dims_t* dims, int shard, const tpla_bf16* latent_raw,
                         const tpla_bf16* kpe_new, int transform, const float* R_dense, const float* norm_weight,
                         float eps, const int32_t* positions, const int32_t* block_table,
                         tpla_bf16* ckv_shard_cache, tpla_bf16* kpe_cache, void* stream) {
    if (dims && (shard < 0 || shard >= dims->g)) return TPLA_ERR_INVALID_ARG;
    return run_append(dims, shard, latent_raw, kpe_new, transform, R_dense, norm_weight, eps, positions, block_table,
                      ckv_shard_cache, kpe_cache, stream);
}

int tpla_check_device_status(void* stream) {
    unsigned* status = nullptr;
    int st = device_info(&status, nullptr);
    if (st) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return TPLA_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpy(&v, status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TPLA_ERR_CUDA;
    const unsigned zero = 0;
    if (cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return TPLA_ERR_CUDA;
    if (v & kStatusTimeout) return TPLA_ERR_TIMEOUT;
    if (v & kStatusIndex) return TPLA_ERR_INDEX;
    return TPLA_OK;
}

int tpla_set_option(int option, int value) {
    switch (option) {
        case TPLA_OPT_ATTENTION_KERNEL:
            if (value < 0 || value > 2) return TPLA_ERR_INVALID_ARG;
            g_opt_kernel = value; return TPLA_OK;
        case TPLA_OPT_MAX_WORKERS:
            if (value < 0) return TPLA_ERR_INVALID_ARG;
            g_opt_max_workers = value; return TPLA_OK;
        case TPLA_OPT_WAIT_LIMIT:
            if (value < 0) return TPLA_ERR_INVALID_ARG;
            g_opt_wait_limit = value; return TPLA_OK;
        case TPLA_OPT_DEBUG_STALL:
            if (value < 0 || value > 1) return TPLA_ERR_INVALID_ARG;
            g_opt_debug_stall = value; return TPLA_OK;
        case TPLA_OPT_TILE_TOKENS:
            if (!(value == 0 || value == 64 || value == 128)) return TPLA_ERR_INVALID_ARG;
            g_opt_tile_tokens = value; return TPLA_OK;
    }
    return TPLA_ERR_INVALID_ARG;
}

int tpla_get_option(int option) {
    switch (option) {
        case TPLA_OPT_ATTENTION_KERNEL: return g_opt_kernel;
        case TPLA_OPT_MAX_WORKERS: return g_opt_max_workers;
        case TPLA_OPT_WAIT_LIMIT: return g_opt_wait_limit;
        case TPLA_OPT_DEBUG_STALL: return g_opt_debug_stall;
        case TPLA_OPT_LAST_ATTENTION_KERNEL: return g_last_kernel;
        case TPLA_OPT_TILE_TOKENS: return g_opt_tile_tokens;
    }
    return -1;
}

const char* tpla_version(void) { return "tpla-b200 0.1 (sm_100a)"; }

}  // extern "C"

// ---------------------------------------------------------------- decode without allocation
//
// For callers that cannot allocate device memory at all: code that runs where
// cudaMalloc is off limits (inside a custom allocator or memory-pool callback,
// under a framework that owns every byte of device memory and hands out
// nothing, or in a hard real-time loop where an allocation may block), and
// that therefore cannot provide a workspace.  tpla_decode_static does what
// tpla_decode does with its scratch in one fixed, file-scope device array.
namespace tpla {
namespace {

constexpr size_t kStaticScratchBytes = 32ull << 20;      // 32 MiB, held by every GPU that loads the library
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_static_mutex;
void* g_static_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once per device
// (the array's name in host code is only a host-side handle, not a device address).
int static_scratch(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return TPLA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return TPLA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_mutex);
    if (!g_static_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || ptr == nullptr) return TPLA_ERR_CUDA;
        g_static_ptr[dev] = ptr;
    }
    *out = g_static_ptr[dev];
    return TPLA_OK;
}

}  // namespace
}  // namespace tpla

extern "C" int tpla_decode_static(const tpla_dims_t* dims, const tpla_bf16* q, const tpla_bf16* q_pe,
                                  const tpla_bf16* ckv, const tpla_bf16* kpe, const int32_t* block_table,
                                  const int32_t* seq_lens, const tpla_bf16* w_uv, float* out, void* stream) {
    int st = check_dims(dims);
    if (st) return st;
    if (dims->B == 0) return TPLA_OK;
    if (!q || !q_pe || !ckv || !kpe || !seq_lens || !out) return TPLA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(q_pe) || !aligned16(ckv) || !aligned16(kpe) || !aligned16(seq_lens) ||
        !aligned16(out))
        return TPLA_ERR_INVALID_ARG;
    if (block_table && !aligned16(block_table)) return TPLA_ERR_INVALID_ARG;
    if (w_uv && !aligned16(w_uv)) return TPLA_ERR_INVALID_ARG;
    if (!block_table && (long long)dims->B * dims->max_pages_per_seq > dims->num_pages) return TPLA_ERR_INVALID_ARG;
    // partial slots that fit next to the header and the log-sum-exp block
    const size_t head = 256 + ws_lse_bytes(dims) + 256;
    if (head >= kStaticScratchBytes) return TPLA_ERR_WORKSPACE;
    const size_t slot_bytes = (size_t)dims->H * (size_t)(dims->L / dims->g) * sizeof(float);
    const long long max_slots = (long long)((kStaticScratchBytes - head) / slot_bytes);
    const long long fixed = (long long)dims->B * dims->g;          // one slot per (sequence, shard)
    if (max_slots - fixed < 1) return TPLA_ERR_WORKSPACE;          // beyond the static scratch, even with one worker
    void* scratch = nullptr;
    if ((st = static_scratch(&scratch))) return st;
    Plan p;
    if ((st = make_plan(dims, -1, &p))) return st;
    if (p.W > max_slots - fixed) p.W = (int)(max_slots - fixed);  // fewer split-KV workers, same result
    // (W + B*g) partial slots follow the log-sum-exp block, which carve() sizes for kMaxWorkers + B*g
    Workspace w = carve(scratch, dims);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((st = launch_attention(p, q, q_pe, ckv, kpe, block_table, seq_lens, w, s))) return st;
    cudaError_t e = launch_combine(p, seq_lens, reinterpret_cast<const __nv_bfloat16*>(w_uv), out, w, s);
    return e == cudaSuccess ? TPLA_OK : TPLA_ERR_CUDA;
}
