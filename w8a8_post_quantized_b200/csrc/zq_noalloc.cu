// zq_noalloc.cu -- a variant of the requantizing W8A8 linear that needs no
// caller-supplied scratch memory and allocates none.
//
// The requantizing linear (zq_w8a8_linear with ZQ_OUT_I8_REQUANT) needs
// scratch: the fp32 epilogue output of the whole row block and a per-token
// absmax word, because the new per-token scale depends on every output
// feature of the token.  Normally the caller passes that scratch as the
// workspace.  Some callers cannot obtain device memory on their own: code
// that runs inside a host framework which owns every device allocation and
// hands its plugins no workspace, and latency-critical serving loops where a
// cudaMalloc (which may synchronize the device) is not allowed after start-up.
// For them this file keeps the scratch in one fixed array in device memory
// that the library owns; the library's other entry points do not touch it.
//
// The array is a file-scope __device__ variable: every GPU that loads the
// library holds ZQ_NOALLOC_SCRATCH_BYTES of device memory for it until the
// process exits.  Host code cannot use its name as a device address, so the
// first call on each device looks the address up with cudaGetSymbolAddress
// (with that device current) and caches it for the life of the process, so
// the entry point must not be used on a device after cudaDeviceReset of it
// (the module, and with it the array, may then be loaded at a new address).
#include <mutex>

#include "zq_internal.cuh"

namespace zq {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[ZQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDev = 64;
std::mutex g_mu;
unsigned char* g_addr[kMaxDev];  // device address of the array, per device

// Once per device, with that device current: the array's device address.
int scratch_address(unsigned char** out) {
    int dev = -1;
    int rc = cuda_status(cudaGetDevice(&dev));
    if (rc) return rc;
    if (dev < 0 || dev >= kMaxDev) return ZQ_ERR_DEVICE;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        if ((rc = cuda_status(cudaGetSymbolAddress(&p, g_noalloc_scratch)))) return rc;
        g_addr[dev] = static_cast<unsigned char*>(p);
    }
    *out = g_addr[dev];
    return ZQ_OK;
}

inline size_t round256(size_t v) { return (v + 255) / 256 * 256; }
inline bool aligned(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

}  // namespace
}  // namespace zq

using namespace zq;

extern "C" int zq_w8a8_linear_requant_noalloc(const int8_t* xq, const float* s_tok, int64_t T,
                                              int64_t K, const int8_t* Wq, const float* s_grp,
                                              int64_t N, int64_t group_rows, const float* bias,
                                              int act, int8_t* y, float* s_tok_out, void* stream) {
    if (!xq || !s_tok || !Wq || !s_grp || !y || !s_tok_out) return ZQ_ERR_NULL;
    if (act != ZQ_ACT_NONE && act != ZQ_ACT_GELU) return ZQ_ERR_DTYPE;
    if (T <= 0 || K <= 0 || N <= 0 || group_rows <= 0) return ZQ_ERR_SHAPE;
    if (K % 16 != 0 || N % 16 != 0 || N % group_rows != 0) return ZQ_ERR_SHAPE;
    if (T > (1 << 30) || N > (1 << 30)) return ZQ_ERR_SHAPE;
    if (K > ZQ_MAX_K) return ZQ_ERR_OVERFLOW;
    if (!aligned(xq, 16) || !aligned(Wq, 16) || !aligned(y, 16) || !aligned(s_tok, 4) ||
        !aligned(s_grp, 4) || !aligned(s_tok_out, 4) || (bias && !aligned(bias, 4)))
        return ZQ_ERR_ALIGN;
    // scratch layout: [absmax words, T x 4 bytes][fp32 epilogue output, T x N x 4 bytes]
    const size_t amax_bytes = round256((size_t)T * 4);
    const size_t h_bytes = (size_t)T * (size_t)N * sizeof(float);
    if (amax_bytes + h_bytes > (size_t)ZQ_NOALLOC_SCRATCH_BYTES) return ZQ_ERR_SCRATCH;

    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    unsigned char* scratch = nullptr;
    if ((rc = scratch_address(&scratch))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

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
    a.out_kind = ZQ_OUT_I8_REQUANT;
    a.y = y;
    a.amax_ws = reinterpret_cast<uint32_t*>(scratch);
    a.h_ws = reinterpret_cast<float*>(scratch + amax_bytes);
    // the array keeps the previous call's contents: the absmax words must start at 0
    if ((rc = cuda_status(cudaMemsetAsync(a.amax_ws, 0, (size_t)T * 4, st)))) return rc;
    if ((rc = launch_w8a8_gemm(a, di, st))) return rc;
    return launch_requant_rows(a.h_ws, T, N, a.amax_ws, y, s_tok_out, di, st);
}
