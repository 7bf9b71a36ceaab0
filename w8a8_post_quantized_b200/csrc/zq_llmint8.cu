// zq_llmint8.cu -- the LLM.int8() mixed-precision decomposition around the
// W8A8 linear: outlier column selection, the LayerNorm parameters that zero
// those columns for the INT8 part, and the fp16 operands of the outlier part.
//
// Source: "探秘Transformer系列之（36）— 大模型量化方案" §1.1 (LLM.int8()): the
// feature columns of the input holding a value above the threshold alpha
// (6.0) form the outlier set O; X[:, O] and the matching weights are
// multiplied in FP16, the other columns are quantized (absmax per token of X,
// per output of W) for the INT8 product, and the dequantized INT8 result and
// the FP16 result are added.  Here: a column is an outlier when its absmax
// over the batch (zq_smooth_calibrate) is >= alpha; at most
// ZQ_LLMINT8_MAX_OUTLIERS columns, the lowest indices, are decomposed; the
// INT8 part is the unchanged LayerNorm + quantizer fed gamma and beta that are
// zero on those columns; the outlier product is added in the GEMM epilogue
// before bias and activation.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int kMaxOut = ZQ_LLMINT8_MAX_OUTLIERS;
constexpr int kSelThreads = 1024;

// One CTA: thread t scans a contiguous range of columns; a block-wide scan of
// the per-thread counts orders the outliers by column index.  Writes the
// first kMaxOut indices (-1 past the count), the total count, and gamma/beta
// with zeros on the decomposed columns.
__global__ void __launch_bounds__(kSelThreads)
llmint8_select_kernel(const float* __restrict__ amax, int K, float threshold, const float* __restrict__ gamma,
                      const float* __restrict__ beta, int32_t* __restrict__ idx, int32_t* __restrict__ count,
                      float* __restrict__ gamma_m, float* __restrict__ beta_m) {
    __shared__ int warp_tot[kSelThreads / 32];
    griddep_wait();  // writes parameters: successors start only at completion
    const int per = (K + kSelThreads - 1) / kSelThreads;
    const int j0 = min(K, (int)threadIdx.x * per), j1 = min(K, j0 + per);
    int local = 0;
    for (int j = j0; j < j1; ++j) local += amax[j] >= threshold ? 1 : 0;
    // exclusive scan over the block
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = warp_tot[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, w, o);
            if (lane >= o) w += v;
        }
        warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    int rank = incl - local + (warp > 0 ? warp_tot[warp - 1] : 0);
    for (int j = j0; j < j1; ++j) {
        const bool out = amax[j] >= threshold;
        const bool decomposed = out && rank < kMaxOut;
        if (decomposed) idx[rank] = j;
        if (gamma_m) gamma_m[j] = decomposed ? 0.0f : gamma[j];
        if (beta_m) beta_m[j] = decomposed ? 0.0f : (beta ? beta[j] : 0.0f);
        rank += out ? 1 : 0;
    }
    const int total = warp_tot[kSelThreads / 32 - 1];
    if (threadIdx.x < kMaxOut && (int)threadIdx.x >= total) idx[threadIdx.x] = -1;
    if (threadIdx.x == 0) *count = total;
}

template <typename Tin>
__device__ __forceinline__ float act_at(const Tin* p);
template <>
__device__ __forceinline__ float act_at<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float act_at<uint16_t>(const uint16_t* p) {
    return __uint_as_float((uint32_t)__ldg(reinterpret_cast<const unsigned short*>(p)) << 16);
}

// The decomposed columns of the LayerNorm output as fp16 [T, 8] (zeros past
// the count): one warp per row computes the row's mean and biased variance
// (two passes, fp32), then lane k < 8 evaluates column idx[k].
template <typename Tin>
__global__ void __launch_bounds__(256)
llmint8_outlier_act_kernel(const Tin* __restrict__ x, int64_t T, int K, const float* __restrict__ gamma,
                           const float* __restrict__ beta, float eps, const int32_t* __restrict__ idx,
                           const int32_t* __restrict__ count, uint16_t* __restrict__ xo) {
    griddep_wait();
    griddep_launch_dependents();
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T) return;
    const int n = min(*count, kMaxOut);
    const Tin* xr = x + t * K;
    float s = 0.0f;
    for (int j = lane; j < K; j += 32) s += act_at(xr + j);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
    const float mean = s / (float)K;
    float q = 0.0f;
    for (int j = lane; j < K; j += 32) {
        const float d = act_at(xr + j) - mean;
        q = fmaf(d, d, q);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
    const float rstd = rsqrtf(q / (float)K + eps);
    if (lane < kMaxOut) {
        float y = 0.0f;
        if (lane < n) {
            const int j = idx[lane];
            y = fmaf((act_at(xr + j) - mean) * rstd, gamma[j], beta ? beta[j] : 0.0f);
        }
        xo[t * kMaxOut + lane] = __half_as_ushort(__float2half_rn(y));
    }
}

// The decomposed columns of the fp32 weights as fp16 [N, 8] (zeros past the count).
__global__ void __launch_bounds__(256)
llmint8_outlier_weights_kernel(const float* __restrict__ W, int64_t N, int64_t K, const int32_t* __restrict__ idx,
                               const int32_t* __restrict__ count, uint16_t* __restrict__ wo) {
    griddep_wait();  // writes weights: successors start only at completion
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= N * kMaxOut) return;
    const int64_t o = i / kMaxOut;
    const int k = (int)(i % kMaxOut);
    const int n = min(*count, kMaxOut);
    const float w = k < n ? __ldg(W + o * K + idx[k]) : 0.0f;
    wo[i] = __half_as_ushort(__float2half_rn(w));
}

template <typename Kern, typename... Args>
int launch_plain(Kern kern, dim3 grid, dim3 block, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

}  // namespace

int launch_llmint8_select(const float* amax, int64_t K, float threshold, const float* gamma, const float* beta,
                          int32_t* idx, int32_t* count, float* gamma_m, float* beta_m, cudaStream_t st) {
    return launch_plain(llmint8_select_kernel, dim3(1), dim3(kSelThreads), st, amax, (int)K, threshold, gamma, beta,
                        idx, count, gamma_m, beta_m);
}

int launch_llmint8_outlier_act(const void* x, int x_dtype, int64_t T, int64_t K, const float* gamma,
                               const float* beta, float eps, const int32_t* idx, const int32_t* count, uint16_t* xo,
                               cudaStream_t st) {
    const dim3 grid((unsigned)((T + 7) / 8)), block(256);
    if (x_dtype == ZQ_BF16)
        return launch_plain(llmint8_outlier_act_kernel<uint16_t>, grid, block, st, static_cast<const uint16_t*>(x), T,
                            (int)K, gamma, beta, eps, idx, count, xo);
    return launch_plain(llmint8_outlier_act_kernel<float>, grid, block, st, static_cast<const float*>(x), T, (int)K,
                        gamma, beta, eps, idx, count, xo);
}

int launch_llmint8_outlier_weights(const float* W, int64_t N, int64_t K, const int32_t* idx, const int32_t* count,
                                   uint16_t* wo, cudaStream_t st) {
    const int64_t total = N * kMaxOut;
    return launch_plain(llmint8_outlier_weights_kernel, dim3((unsigned)((total + 255) / 256)), dim3(256), st, W, N, K,
                        idx, count, wo);
}

}  // namespace zq
