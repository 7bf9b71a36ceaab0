// zq_noalloc.cu -- a variant of the requantizing W8A8 linear that needs no
// caller-supplied scratch memory and allocates none.
//
// The requantizing linear (zq_w8a8_linear with ZQ_OUT_I8_REQUANT) needs
// scratch for most shapes, because the new per-token scale depends on every
// output feature of the token: per-token absmax words and per-row-block
// arrival counters (rows wider than 4096 features), or the fp32 epilogue
// output and the absmax words (at most 64 tokens).  Normally the caller
// passes that scratch as the workspace.  Some callers cannot obtain device memory on their own: code
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
    // The least scratch any route could need for this shape: none for at most
    // 4096 features (the cluster kernel), a word per row and per row block for
    // wider rows (the grid kernel), the fp32 output for at most 64 tokens (the
    // scratch route).  Larger than the array: refused before any device call.
    const size_t least = T <= 64 ? requant_scratch_route_bytes(T, N) : N <= 4096 ? 0 : requant_grid_scratch_bytes(T);
    if (least > (size_t)ZQ_NOALLOC_SCRATCH_BYTES) return ZQ_ERR_SCRATCH;

    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    unsigned char* scratch = nullptr;
    if ((rc = scratch_address(&scratch))) return rc;

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
    a.s_tok_out = s_tok_out;
    // the same routes as zq_w8a8_linear, with the array as their scratch; each
    // route clears what must start at zero (the array keeps the previous
    // call's contents)
    return run_requant(a, scratch, (size_t)ZQ_NOALLOC_SCRATCH_BYTES, ZQ_ERR_SCRATCH, di,
                       static_cast<cudaStream_t>(stream));
}
