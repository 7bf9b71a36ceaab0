// zq_api.cu -- the C ABI declared in include/zq.h: argument validation (all
// of it on the host, before anything is enqueued), per-device facts, the
// device status word used by bounded waits, and the entry points.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "zq_internal.cuh"

#define ZQ_VERSION 100  // 0.1.0

namespace zq {

// Device status word: bounded waits record the site of an expired wait here.
__device__ int g_status_word;

static thread_local char t_last_error[256] = "no error";
static std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

std::mutex& launch_cache_mutex() {
    static std::mutex mu;
    return mu;
}

int requant_route() {
    static const int route = [] {
        const char* v = getenv("ZQ_REQUANT_ROUTE");
        if (!v) return 0;
        if (!strcmp(v, "cluster")) return 1;
        if (!strcmp(v, "grid")) return 2;
        if (!strcmp(v, "scratch")) return 3;
        return 0;
    }();
    return route;
}

int even_split_mode() {
    // read on every call (a workspace query and the call it sizes may then
    // disagree; the workspace is optional where this applies, so a call
    // whose workspace is too small takes the other route)
    const char* v = getenv("ZQ_EVEN_SPLIT");
    if (!v) return 0;
    if (!strcmp(v, "off")) return 1;
    if (!strcmp(v, "on")) return 2;
    return 0;
}

int pdl_attr(cudaLaunchAttribute& attr) {
    static const bool off = getenv("ZQ_NO_PDL") != nullptr;
    if (off) return 0;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    return 1;
}

void set_cuda_error(cudaError_t e) {
    snprintf(t_last_error, sizeof(t_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}

int cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return ZQ_OK;
    set_cuda_error(e);
    return ZQ_ERR_CUDA;
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
bool g_have[kMaxDevices];
DeviceInfo g_info[kMaxDevices];
}  // namespace

int device_info(DeviceInfo* out) {
    int dev = -1;
    int rc = cuda_status(cudaGetDevice(&dev));
    if (rc) return rc;
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_have[dev]) {
        DeviceInfo di{};
        if ((rc = cuda_status(cudaDeviceGetAttribute(&di.sm_count, cudaDevAttrMultiProcessorCount, dev))))
            return rc;
        if ((rc = cuda_status(cudaDeviceGetAttribute(&di.major, cudaDevAttrComputeCapabilityMajor, dev))))
            return rc;
        if ((rc = cuda_status(cudaDeviceGetAttribute(&di.minor, cudaDevAttrComputeCapabilityMinor, dev))))
            return rc;
        void* addr = nullptr;
        if ((rc = cuda_status(cudaGetSymbolAddress(&addr, g_status_word)))) return rc;
        di.status_word = static_cast<int*>(addr);
        g_info[dev] = di;
        g_have[dev] = true;
    }
    *out = g_info[dev];
    // sm_100a code only runs on compute capability 10.0 parts
    if (out->major != 10 || out->minor != 0) return ZQ_ERR_DEVICE;
    return ZQ_OK;
}

}  // namespace zq

using namespace zq;

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

int check_rows(const void* x, int x_dtype, int64_t T, int64_t H, const int8_t* q, const float* s_tok) {
    if (!x || !q || !s_tok) return ZQ_ERR_NULL;
    if (x_dtype != ZQ_F32 && x_dtype != ZQ_BF16) return ZQ_ERR_DTYPE;
    if (T <= 0 || H <= 0 || H % 16 != 0 || H > ZQ_MAX_H) return ZQ_ERR_SHAPE;
    if (T > (int64_t)1 << 31) return ZQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(s_tok, 4)) return ZQ_ERR_ALIGN;
    return ZQ_OK;
}

constexpr size_t kWsAlign = 256;
inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

size_t linear_ws_bytes(int64_t T, int64_t K, int64_t N, int out_kind) {
    if (T <= 0 || N <= 0) return 0;
    // the SM count decides which kernels cover the shape; without a usable
    // device assume the scratch route (and no even split)
    int sms = 0;
    DeviceInfo di;
    if (device_info(&di) == ZQ_OK) sms = di.sm_count;
    if (out_kind != ZQ_OUT_I8_REQUANT)  // optional: the partial sums of the few-token even split
        return decode_even_applies(T, K, N, sms) ? round_up(decode_sk_ws_bytes(sms), kWsAlign) : 0;
    return requant_ws_bytes(T, N, sms);
}

int check_linear(const int8_t* xq, const float* s_tok, int64_t T, int64_t K, const int8_t* Wq,
                 const float* s_grp, int64_t N, int64_t G, const float* bias, int act, int out_kind,
                 void* y, float* s_tok_out, void* ws, size_t ws_bytes, bool check_x) {
    if (check_x && (!xq || !s_tok)) return ZQ_ERR_NULL;
    if (!Wq || !s_grp || !y) return ZQ_ERR_NULL;
    if (out_kind < ZQ_OUT_F32 || out_kind > ZQ_OUT_I32_RAW) return ZQ_ERR_DTYPE;
    if (act != ZQ_ACT_NONE && act != ZQ_ACT_GELU) return ZQ_ERR_DTYPE;
    if (out_kind == ZQ_OUT_I32_RAW && (act != ZQ_ACT_NONE || bias)) return ZQ_ERR_DTYPE;
    if (out_kind == ZQ_OUT_I8_REQUANT && !s_tok_out) return ZQ_ERR_NULL;
    if (T <= 0 || K <= 0 || N <= 0 || G <= 0) return ZQ_ERR_SHAPE;
    if (K % 16 != 0 || N % 16 != 0 || N % G != 0) return ZQ_ERR_SHAPE;
    if (T > (1 << 30) || N > (1 << 30)) return ZQ_ERR_SHAPE;
    if (K > ZQ_MAX_K) return ZQ_ERR_OVERFLOW;
    if (check_x && (!aligned(xq, 16) || !aligned(s_tok, 4))) return ZQ_ERR_ALIGN;
    if (!aligned(Wq, 16) || !aligned(y, 16) || !aligned(s_grp, 4)) return ZQ_ERR_ALIGN;
    if ((bias && !aligned(bias, 4)) || (s_tok_out && !aligned(s_tok_out, 4))) return ZQ_ERR_ALIGN;
    if (ws && !aligned(ws, 16)) return ZQ_ERR_ALIGN;
    // required for the requantizing kinds; optional otherwise (the few-token
    // kernels then split K over clusters instead of evenly over all SMs)
    if (out_kind == ZQ_OUT_I8_REQUANT) {
        const size_t need = linear_ws_bytes(T, K, N, out_kind);
        if (need && (!ws || ws_bytes < need)) return ZQ_ERR_WORKSPACE;
    }
    return ZQ_OK;
}

int run_linear(const int8_t* xq, const float* s_tok, int64_t T, int64_t K, const int8_t* Wq,
               const float* s_grp, int64_t N, int64_t G, const float* bias, int act, int out_kind,
               void* y, float* s_tok_out, void* ws, size_t ws_bytes, const DeviceInfo& di, cudaStream_t st) {
    LinearArgs a{};
    a.xq = xq;
    a.s_tok = s_tok;
    a.T = T;
    a.K = K;
    a.Wq = Wq;
    a.s_grp = s_grp;
    a.N = N;
    a.G = G;
    a.bias = bias;
    a.act = act;
    a.out_kind = out_kind;
    a.y = y;
    a.s_tok_out = s_tok_out;
    if (out_kind == ZQ_OUT_I8_REQUANT) return run_requant(a, ws, ws_bytes, ZQ_ERR_WORKSPACE, di, st);
    // few tokens: the even split where it is taken and the workspace holds its partials
    if (decode_even_applies(T, K, N, di.sm_count) && ws && ws_bytes >= decode_sk_ws_bytes(di.sm_count)) {
        const int rc = launch_w8a8_decode_sk(a, ws, ws_bytes, di, st);
        if (rc != ZQ_ERR_SHAPE) return rc;
    }
    return launch_w8a8_gemm(a, di, st);
}

}  // namespace

namespace zq {

size_t requant_scratch_route_bytes(int64_t T, int64_t N) {
    // fp32 [T, N] epilogue output + [T] absmax words
    return round_up((size_t)T * (size_t)N * sizeof(float), kWsAlign) + round_up((size_t)T * 4, kWsAlign);
}

size_t requant_ws_bytes(int64_t T, int64_t N, int sms) {
    const int64_t n_t = (N + 255) / 256;
    const int route = requant_route();
    // T > 64 with at most one column tile per SM: the fused kernels (the
    // cluster kernel needs none, the grid kernel a word per row and per row block)
    if ((route == 0 || route == 2) && T > 64 && sms > 0 && n_t <= sms)
        return round_up(requant_grid_scratch_bytes(T), kWsAlign);
    return requant_scratch_route_bytes(T, N);
}

int run_requant(const LinearArgs& a0, void* ws, size_t ws_bytes, int err_small, const DeviceInfo& di,
                cudaStream_t st) {
    LinearArgs a = a0;
    const int route = requant_route();
    int rc;
    // fused: the row absmax is exchanged inside a thread-block cluster (N <= 4096)
    if (route == 0 || route == 1) {
        rc = launch_w8a8_requant_cluster(a, di, st);
        if (rc != ZQ_ERR_SHAPE) return rc;
    }
    // fused, any width: the row absmax is exchanged through global memory
    if (route == 0 || route == 2) {
        rc = launch_w8a8_requant_grid(a, static_cast<uint32_t*>(ws), ws_bytes, di, st);
        if (rc == ZQ_ERR_WORKSPACE) return err_small;
        if (rc != ZQ_ERR_SHAPE) return rc;
    }
    // otherwise: fp32 epilogue output + row absmax in the scratch, then requantize
    if (!ws || ws_bytes < requant_scratch_route_bytes(a.T, a.N)) return err_small;
    uint8_t* w = static_cast<uint8_t*>(ws);
    a.h_ws = reinterpret_cast<float*>(w);
    a.amax_ws = reinterpret_cast<uint32_t*>(w + round_up((size_t)a.T * a.N * sizeof(float), kWsAlign));
    if ((rc = cuda_status(cudaMemsetAsync(a.amax_ws, 0, (size_t)a.T * 4, st)))) return rc;
    if ((rc = launch_w8a8_gemm(a, di, st))) return rc;
    return launch_requant_rows(a.h_ws, a.T, a.N, a.amax_ws, static_cast<int8_t*>(a.y), a.s_tok_out, di, st);
}

}  // namespace zq

extern "C" {

int zq_version(void) { return ZQ_VERSION; }

uint64_t zq_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* zq_status_string(int status) {
    switch (status) {
        case ZQ_OK: return "ok";
        case ZQ_ERR_NULL: return "required pointer is NULL";
        case ZQ_ERR_SHAPE: return "invalid shape (non-positive, not a multiple of 16, N % G != 0, or too large)";
        case ZQ_ERR_ALIGN: return "misaligned pointer (tensors need 16 bytes, vectors 4 bytes)";
        case ZQ_ERR_OVERFLOW: return "K too large: int32 accumulators could overflow";
        case ZQ_ERR_DTYPE: return "unknown or unsupported dtype / activation / output kind";
        case ZQ_ERR_CUDA: return "CUDA error (see zq_last_cuda_error)";
        case ZQ_ERR_TIMEOUT: return "a bounded device-side wait expired";
        case ZQ_ERR_WORKSPACE: return "workspace missing or too small";
        case ZQ_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
        case ZQ_ERR_SCRATCH: return "problem exceeds the fixed scratch array of the no-allocation entry point";
        default: return "unknown status";
    }
}

const char* zq_last_cuda_error(void) { return t_last_error; }

namespace zq {
namespace {
constexpr int kSiteWatchdogSelftest = 0x7E57;
// One thread waits on an mbarrier that nothing arrives on: the bounded wait
// expires after its limit, records the site in the status word and returns.
__global__ void watchdog_selftest_kernel(int* status) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t b = smem_u32(&bar);
    if (threadIdx.x == 0) {
        mbar_init(b, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(b, 0u, nullptr, status, kSiteWatchdogSelftest);
}
}  // namespace
}  // namespace zq

int zq_watchdog_selftest(void* stream) {
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    count_launch();
    watchdog_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(di.status_word);
    return cuda_status(cudaGetLastError());
}

int zq_device_status(void* stream) {
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    if ((rc = cuda_status(cudaStreamSynchronize(as_stream(stream))))) return rc;
    int word = 0;
    if ((rc = cuda_status(cudaMemcpyFromSymbol(&word, g_status_word, sizeof(int))))) return rc;
    if (word != 0) {
        const int zero = 0;
        if ((rc = cuda_status(cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int))))) return rc;
        snprintf(t_last_error, sizeof(t_last_error), "bounded wait expired at site 0x%x", word);
        return ZQ_ERR_TIMEOUT;
    }
    return ZQ_OK;
}

int zq_quantize_weights(const float* W, int64_t N, int64_t K, int64_t group_rows, int8_t* Wq,
                        float* s_grp, void* stream) {
    if (!W || !Wq || !s_grp) return ZQ_ERR_NULL;
    if (N <= 0 || K <= 0 || group_rows <= 0 || K % 16 != 0 || N % group_rows != 0) return ZQ_ERR_SHAPE;
    if (N > ((int64_t)1 << 40) / K) return ZQ_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(s_grp, 4)) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_quantize_weights(W, N, K, group_rows, Wq, s_grp, di, as_stream(stream));
}

int zq_llmint8_select(const float* amax, int64_t K, float threshold, const float* gamma, const float* beta,
                      int32_t* idx, int32_t* count, float* gamma_m, float* beta_m, void* stream) {
    if (!amax || !idx || !count || !gamma || !gamma_m || !beta_m) return ZQ_ERR_NULL;
    if (K <= 0 || K % 16 != 0 || K > ZQ_MAX_H) return ZQ_ERR_SHAPE;
    if (!aligned(amax, 4) || !aligned(idx, 4) || !aligned(count, 4) || !aligned(gamma, 4) || !aligned(gamma_m, 4) ||
        !aligned(beta_m, 4) || (beta && !aligned(beta, 4)))
        return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_llmint8_select(amax, K, threshold, gamma, beta, idx, count, gamma_m, beta_m, as_stream(stream));
}

int zq_llmint8_outlier_act(const void* x, int x_dtype, int64_t T, int64_t K, const float* gamma, const float* beta,
                           float eps, const int32_t* idx, const int32_t* count, void* xo, void* stream) {
    if (!x || !gamma || !idx || !count || !xo) return ZQ_ERR_NULL;
    if (x_dtype != ZQ_F32 && x_dtype != ZQ_BF16) return ZQ_ERR_DTYPE;
    if (T <= 0 || K <= 0 || K % 16 != 0 || K > ZQ_MAX_H || T > ((int64_t)1 << 31)) return ZQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(xo, 16) || !aligned(gamma, 4) || (beta && !aligned(beta, 4))) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_llmint8_outlier_act(x, x_dtype, T, K, gamma, beta, eps, idx, count, static_cast<uint16_t*>(xo),
                                      as_stream(stream));
}

int zq_llmint8_outlier_weights(const float* W, int64_t N, int64_t K, const int32_t* idx, const int32_t* count,
                               void* wo, void* stream) {
    if (!W || !idx || !count || !wo) return ZQ_ERR_NULL;
    if (N <= 0 || K <= 0 || K % 16 != 0 || N > ((int64_t)1 << 40) / K) return ZQ_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(wo, 16)) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_llmint8_outlier_weights(W, N, K, idx, count, static_cast<uint16_t*>(wo), as_stream(stream));
}

int zq_w8a8_linear_llmint8(const int8_t* xq, const float* s_tok, int64_t T, int64_t K, const int8_t* Wq,
                           const float* s_grp, int64_t N, int64_t group_rows, const float* bias, int act,
                           int out_kind, const void* xo, const void* wo, void* y, void* stream) {
    if (out_kind != ZQ_OUT_F32 && out_kind != ZQ_OUT_BF16) return ZQ_ERR_DTYPE;
    if (!xo || !wo) return ZQ_ERR_NULL;
    if (!aligned(xo, 16) || !aligned(wo, 16)) return ZQ_ERR_ALIGN;
    int rc = check_linear(xq, s_tok, T, K, Wq, s_grp, N, group_rows, bias, act, out_kind, y, nullptr, nullptr, 0,
                          true);
    if (rc) return rc;
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    LinearArgs a{};
    a.xq = xq;
    a.s_tok = s_tok;
    a.T = T;
    a.K = K;
    a.Wq = Wq;
    a.s_grp = s_grp;
    a.N = N;
    a.G = group_rows;
    a.bias = bias;
    a.act = act;
    a.out_kind = out_kind;
    a.y = y;
    return launch_w8a8_gemm_outliers(a, static_cast<const uint16_t*>(xo), static_cast<const uint16_t*>(wo), di,
                                     as_stream(stream));
}

int zq_smooth_calibrate(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                        const float* beta, float eps, float* amax, void* stream) {
    if (!x || !amax) return ZQ_ERR_NULL;
    if (x_dtype != ZQ_F32 && x_dtype != ZQ_BF16) return ZQ_ERR_DTYPE;
    // H <= 32768: the kernel keeps one maximum per channel in shared memory
    if (T <= 0 || H <= 0 || H % 16 != 0 || H > 32768 || T > ((int64_t)1 << 31) - 32) return ZQ_ERR_SHAPE;
    if (!aligned(x, 16) || !aligned(amax, 4) || (gamma && !aligned(gamma, 4)) || (beta && !aligned(beta, 4)))
        return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_smooth_calibrate(x, x_dtype, T, H, gamma, gamma ? beta : nullptr, eps, amax, di, as_stream(stream));
}

int zq_smooth_weights(const float* W, int64_t N, int64_t K, const float* amax, float alpha, const float* gamma,
                      const float* beta, float* W_out, float* gamma_out, float* beta_out, float* s, void* stream) {
    if (!W || !amax || !W_out || !s) return ZQ_ERR_NULL;
    if ((gamma && !gamma_out) || (beta && !beta_out)) return ZQ_ERR_NULL;
    if (!(alpha >= 0.0f && alpha <= 1.0f)) return ZQ_ERR_DTYPE;
    if (N <= 0 || K <= 0 || K % 16 != 0 || N > ((int64_t)1 << 40) / K) return ZQ_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(W_out, 16) || !aligned(s, 16) || !aligned(amax, 4)) return ZQ_ERR_ALIGN;
    if ((gamma && !aligned(gamma, 4)) || (beta && !aligned(beta, 4)) || (gamma_out && !aligned(gamma_out, 4)) ||
        (beta_out && !aligned(beta_out, 4)))
        return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    return launch_smooth_weights(W, N, K, amax, alpha, gamma, beta, W_out, gamma_out, beta_out, s, di,
                                 as_stream(stream));
}

int zq_ln_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                const float* beta, float eps, int8_t* q, float* s_tok, void* stream) {
    int rc = check_rows(x, x_dtype, T, H, q, s_tok);
    if (rc) return rc;
    if (!gamma || !beta) return ZQ_ERR_NULL;
    if (!aligned(gamma, 16) || !aligned(beta, 16)) return ZQ_ERR_ALIGN;
    if (!(eps >= 0.0f)) return ZQ_ERR_SHAPE;
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    return launch_ln_quant(x, x_dtype, T, H, gamma, beta, eps, q, s_tok, di, as_stream(stream));
}

int zq_act_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* bias, int act,
                 int8_t* q, float* s_tok, void* stream) {
    int rc = check_rows(x, x_dtype, T, H, q, s_tok);
    if (rc) return rc;
    if (act != ZQ_ACT_NONE && act != ZQ_ACT_GELU) return ZQ_ERR_DTYPE;
    if (bias && !aligned(bias, 16)) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    return launch_act_quant(x, x_dtype, T, H, bias, act, q, s_tok, di, as_stream(stream));
}

size_t zq_w8a8_linear_workspace(int64_t T, int64_t K, int64_t N, int out_kind) {
    return linear_ws_bytes(T, K, N, out_kind);
}

int zq_w8a8_linear(const int8_t* xq, const float* s_tok, int64_t T, int64_t K, const int8_t* Wq,
                   const float* s_grp, int64_t N, int64_t group_rows, const float* bias, int act,
                   int out_kind, void* y, float* s_tok_out, void* workspace, size_t workspace_bytes,
                   void* stream) {
    int rc = check_linear(xq, s_tok, T, K, Wq, s_grp, N, group_rows, bias, act, out_kind, y, s_tok_out,
                          workspace, workspace_bytes, true);
    if (rc) return rc;
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    return run_linear(xq, s_tok, T, K, Wq, s_grp, N, group_rows, bias, act, out_kind, y, s_tok_out,
                      workspace, workspace_bytes, di, as_stream(stream));
}

size_t zq_linear_block_workspace(int64_t T, int64_t K, int64_t N, int out_kind) {
    if (T <= 0 || K <= 0) return 0;
    return round_up((size_t)T * (size_t)K, kWsAlign) + round_up((size_t)T * 4, kWsAlign) +
           linear_ws_bytes(T, K, N, out_kind);
}

int zq_linear_block(const void* x, int x_dtype, int64_t T, int64_t K, const float* gamma,
                    const float* beta, float eps, const int8_t* Wq, const float* s_grp, int64_t N,
                    int64_t group_rows, const float* bias, int act, int out_kind, void* y,
                    float* s_tok_out, void* workspace, size_t workspace_bytes, void* stream) {
    if (!x) return ZQ_ERR_NULL;
    if (x_dtype != ZQ_F32 && x_dtype != ZQ_BF16) return ZQ_ERR_DTYPE;
    if (T <= 0 || K <= 0 || K > ZQ_MAX_H) return ZQ_ERR_SHAPE;
    if (gamma && !beta) return ZQ_ERR_NULL;
    if (gamma && (!aligned(gamma, 16) || !aligned(beta, 16))) return ZQ_ERR_ALIGN;
    if (gamma && !(eps >= 0.0f)) return ZQ_ERR_SHAPE;
    if (!aligned(x, 16)) return ZQ_ERR_ALIGN;
    const size_t need = zq_linear_block_workspace(T, K, N, out_kind);
    if (!workspace || workspace_bytes < need) return ZQ_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return ZQ_ERR_ALIGN;
    uint8_t* w = static_cast<uint8_t*>(workspace);
    int8_t* xq = reinterpret_cast<int8_t*>(w);
    float* s_tok = reinterpret_cast<float*>(w + round_up((size_t)T * K, kWsAlign));
    uint8_t* lin_ws = w + round_up((size_t)T * K, kWsAlign) + round_up((size_t)T * 4, kWsAlign);
    const size_t lin_bytes = workspace_bytes - (size_t)(lin_ws - w);
    int rc = check_linear(xq, s_tok, T, K, Wq, s_grp, N, group_rows, bias, act, out_kind, y, s_tok_out,
                          lin_ws, lin_bytes, false);
    if (rc) return rc;
    DeviceInfo di;
    if ((rc = device_info(&di))) return rc;
    cudaStream_t st = as_stream(stream);
    if (gamma) rc = launch_ln_quant(x, x_dtype, T, K, gamma, beta, eps, xq, s_tok, di, st);
    else rc = launch_act_quant(x, x_dtype, T, K, nullptr, ZQ_ACT_NONE, xq, s_tok, di, st);
    if (rc) return rc;
    return run_linear(xq, s_tok, T, K, Wq, s_grp, N, group_rows, bias, act, out_kind, y, s_tok_out,
                      lin_ws, lin_bytes, di, st);
}

}  // extern "C"
