// zq_smooth.cu -- SmoothQuant offline steps: calibration of the per-channel
// absmax of a linear's input activation, the smoothing factors, and their
// fold into the preceding LayerNorm's gamma/beta and into the weights.
//
// Sources: "探秘Transformer系列之（36）— 大模型量化方案" §1.3 (a per-channel
// smoothing factor s chosen offline; Y = (X diag(s)^-1)(diag(s) W) leaves the
// output unchanged while the activations shrink and the weights grow) and
// "SmoothQuant技术解析：大模型INT8量化的突破与实践" §2.2 (s makes the channel
// maxima of the smoothed activation alike), §3 (per-channel max |X| over
// calibration batches; the weights are transformed offline, then quantized).
// The factor is the SmoothQuant paper's balance rule
//   s_j = amax_j^alpha / wmax_j^(1 - alpha),  s_j >= 1e-5,
// with s_j = 1 for a channel whose activation or weight absmax is 0.  The
// activation side diag(s)^-1 is folded into gamma and beta, so the online
// kernels run unchanged on the smoothed parameters.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int kCalibRows = 32;    // rows per block (LN statistics: four rows per warp)
constexpr int kCalibThreads = 256;

// 16-byte vectors of the activation: 8 bf16 or 4 fp32 values.
template <typename Tin>
struct Vec;
template <>
struct Vec<float> {
    static constexpr int N = 4;
    static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(p));
        v[0] = t.x;
        v[1] = t.y;
        v[2] = t.z;
        v[3] = t.w;
    }
};
template <>
struct Vec<uint16_t> {
    static constexpr int N = 8;
    static __device__ __forceinline__ void load(const uint16_t* p, float (&v)[8]) {
        const uint4 t = __ldg(reinterpret_cast<const uint4*>(p));
        const uint32_t w[4] = {t.x, t.y, t.z, t.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_lo(w[i]);
            v[2 * i + 1] = bf16_hi(w[i]);
        }
    }
};

// Running per-channel absmax.  Persistent CTAs walk blocks of kCalibRows
// rows.  With LN the activation is the LayerNorm output (two-pass fp32 mean
// and biased variance per row, one warp per row, eps inside the square root),
// else x itself.  Rows are read as 16-byte vectors of VN channels.  When a row
// has at most 256 vectors, thread t owns vector t % nv of every (t / nv)-th
// row lane and keeps its maxima in registers across all of the CTA's rows;
// otherwise a thread folds each block's rows for its vectors into a
// shared-memory maximum.  Either way the CTA ends with one global atomic max
// per channel (values are >= 0, so their bit patterns order like the floats).
template <typename Tin, bool LN>
__global__ void __launch_bounds__(kCalibThreads)
smooth_calib_kernel(const Tin* __restrict__ x, int T, int H, const float* __restrict__ gamma,
                    const float* __restrict__ beta, float eps, uint32_t* __restrict__ amax_bits) {
    constexpr int VN = Vec<Tin>::N;
    extern __shared__ uint32_t s_cmax[];  // [H] when nv > kCalibThreads, else [kCalibThreads / nv * ... ] reuse
    __shared__ float s_mean[kCalibRows], s_rstd[kCalibRows];
    const int nv = H / VN;  // vectors per row (H % 16 == 0)
    const int nblocks = (T + kCalibRows - 1) / kCalibRows;
    const bool regs = nv <= kCalibThreads;
    const int lanes = regs ? kCalibThreads / nv : 1;  // row lanes per vector
    const int my_v = threadIdx.x % nv, my_lane = threadIdx.x / nv;
    griddep_wait();
    griddep_launch_dependents();
    for (int i = threadIdx.x; i < H; i += kCalibThreads) s_cmax[i] = 0u;
    float g[VN], b[VN], m[VN];
#pragma unroll
    for (int e = 0; e < VN; ++e) {
        const int c = my_v * VN + e;
        g[e] = (LN && regs && my_v < nv) ? __ldg(gamma + c) : 1.0f;
        b[e] = (LN && regs && beta && my_v < nv) ? __ldg(beta + c) : 0.0f;
        m[e] = 0.0f;
    }
    __syncthreads();
    for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
        const int r0 = blk * kCalibRows;
        const int rows = min(kCalibRows, T - r0);
        if constexpr (LN) {
            const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
            for (int r = warp; r < rows; r += kCalibThreads / 32) {
                const Tin* xr = x + (int64_t)(r0 + r) * H;
                float s = 0.0f;
                for (int i = lane; i < nv; i += 32) {
                    float v[VN];
                    Vec<Tin>::load(xr + i * VN, v);
#pragma unroll
                    for (int e = 0; e < VN; ++e) s += v[e];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
                const float mean = s / (float)H;
                float q = 0.0f;
                for (int i = lane; i < nv; i += 32) {
                    float v[VN];
                    Vec<Tin>::load(xr + i * VN, v);
#pragma unroll
                    for (int e = 0; e < VN; ++e) {
                        const float d = v[e] - mean;
                        q = fmaf(d, d, q);
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) q += __shfl_xor_sync(0xFFFFFFFFu, q, o);
                if (lane == 0) {
                    s_mean[r] = mean;
                    s_rstd[r] = rsqrtf(q / (float)H + eps);
                }
            }
            __syncthreads();
        }
        if (regs) {
            if (my_lane < lanes) {
                for (int r = my_lane; r < rows; r += lanes) {
                    float v[VN];
                    Vec<Tin>::load(x + (int64_t)(r0 + r) * H + my_v * VN, v);
#pragma unroll
                    for (int e = 0; e < VN; ++e) {
                        const float a = LN ? fmaf((v[e] - s_mean[r]) * s_rstd[r], g[e], b[e]) : v[e];
                        m[e] = fmaxf(m[e], fabsf(a));
                    }
                }
            }
        } else {
            for (int i = threadIdx.x; i < nv; i += kCalibThreads) {
                float mm[VN];
#pragma unroll
                for (int e = 0; e < VN; ++e) mm[e] = 0.0f;
                for (int r = 0; r < rows; ++r) {
                    float v[VN];
                    Vec<Tin>::load(x + (int64_t)(r0 + r) * H + i * VN, v);
#pragma unroll
                    for (int e = 0; e < VN; ++e) {
                        const int c = i * VN + e;
                        const float a =
                            LN ? fmaf((v[e] - s_mean[r]) * s_rstd[r], __ldg(gamma + c), beta ? __ldg(beta + c) : 0.0f)
                               : v[e];
                        mm[e] = fmaxf(mm[e], fabsf(a));
                    }
                }
#pragma unroll
                for (int e = 0; e < VN; ++e) atomicMax(s_cmax + i * VN + e, __float_as_uint(mm[e]));
            }
        }
        if constexpr (LN) __syncthreads();  // s_mean / s_rstd are rewritten by the next block
    }
    if (regs && my_lane < lanes) {
#pragma unroll
        for (int e = 0; e < VN; ++e) atomicMax(s_cmax + my_v * VN + e, __float_as_uint(m[e]));
    }
    __syncthreads();
    for (int i = threadIdx.x; i < H; i += kCalibThreads) atomicMax(amax_bits + i, s_cmax[i]);
}

// wmax[j] = max over rows of |W[o, j]| (W fp32 [N, K]); a thread owns four
// consecutive columns (16-byte loads) of a slab of kColRows rows.
constexpr int kColRows = 16;
__global__ void __launch_bounds__(256)
weight_col_absmax_kernel(const float* __restrict__ W, int64_t N, int64_t K, uint32_t* __restrict__ wmax_bits) {
    griddep_wait();
    griddep_launch_dependents();
    const int64_t j4 = (int64_t)blockIdx.x * 256 + threadIdx.x;  // float4 column index
    if (j4 >= K / 4) return;
    const int64_t o0 = (int64_t)blockIdx.y * kColRows;
    const int64_t o1 = min(N, o0 + kColRows);
    float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t o = o0; o < o1; ++o) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(W + o * K) + j4);
        m.x = fmaxf(m.x, fabsf(w.x));
        m.y = fmaxf(m.y, fabsf(w.y));
        m.z = fmaxf(m.z, fabsf(w.z));
        m.w = fmaxf(m.w, fabsf(w.w));
    }
    atomicMax(wmax_bits + 4 * j4, __float_as_uint(m.x));
    atomicMax(wmax_bits + 4 * j4 + 1, __float_as_uint(m.y));
    atomicMax(wmax_bits + 4 * j4 + 2, __float_as_uint(m.z));
    atomicMax(wmax_bits + 4 * j4 + 3, __float_as_uint(m.w));
}

// s_j from the activation and weight maxima (the latter in s on entry, so the
// factor overwrites it in place), and the LayerNorm fold gamma/s, beta/s.
// The powers run in double; the factor is rounded once to fp32.
__global__ void __launch_bounds__(256)
smooth_factor_kernel(const float* __restrict__ amax, float* s, int64_t K, double alpha, const float* gamma,
                     const float* beta, float* gamma_out, float* beta_out) {
    griddep_wait();  // writes weights / parameters: successors start only at completion
    const int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x;
    if (j >= K) return;
    const float a = amax[j], w = s[j];
    float f = 1.0f;
    if (a != 0.0f && w != 0.0f) {
        f = (float)(pow((double)a, alpha) / pow((double)w, 1.0 - alpha));
        f = f < 1e-5f ? 1e-5f : f;
    }
    s[j] = f;
    // IEEE single divisions: equal to the fp64 quotient rounded once to fp32
    if (gamma) gamma_out[j] = __fdiv_rn(gamma[j], f);
    if (beta) beta_out[j] = __fdiv_rn(beta[j], f);
}

// W_out[o, j] = W[o, j] * s[j] (one fp32 rounding of the exact product).
__global__ void __launch_bounds__(256)
smooth_fold_kernel(const float* W, int64_t N, int64_t K, const float* __restrict__ s, float* W_out) {
    griddep_wait();  // writes weights / parameters: successors start only at completion
    const int64_t n4 = N * K / 4;  // K % 16 == 0: rows are whole float4s
    const int64_t k4 = K / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4; i += (int64_t)gridDim.x * blockDim.x) {
        const float4 w = reinterpret_cast<const float4*>(W)[i];
        const float4 f = __ldg(reinterpret_cast<const float4*>(s) + i % k4);
        reinterpret_cast<float4*>(W_out)[i] = make_float4(__fmul_rn(w.x, f.x), __fmul_rn(w.y, f.y),
                                                          __fmul_rn(w.z, f.z), __fmul_rn(w.w, f.w));
    }
}

template <typename K, typename... Args>
int launch_smem(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t st, Args... args) {
    // the kernel's static arrays count against the same 48 KB default, so
    // raise the dynamic limit whenever the request comes near it
    if (smem > 32 * 1024) {
        const int rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
        if (rc) return rc;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, args...));
}

template <typename K, typename... Args>
int launch(K kern, dim3 grid, dim3 block, cudaStream_t st, Args... args) {
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

int launch_smooth_calibrate(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                            const float* beta, float eps, float* amax, const DeviceInfo& di, cudaStream_t st) {
    const int64_t nblocks = (T + kCalibRows - 1) / kCalibRows;
    const dim3 grid((unsigned)(nblocks < di.sm_count ? nblocks : di.sm_count)), block(kCalibThreads);
    const size_t smem = (size_t)H * sizeof(uint32_t);  // per-channel maxima of the CTA
    uint32_t* bits = reinterpret_cast<uint32_t*>(amax);
    if (x_dtype == ZQ_BF16) {
        const uint16_t* xb = static_cast<const uint16_t*>(x);
        return gamma ? launch_smem(smooth_calib_kernel<uint16_t, true>, grid, block, smem, st, xb, (int)T, (int)H,
                                   gamma, beta, eps, bits)
                     : launch_smem(smooth_calib_kernel<uint16_t, false>, grid, block, smem, st, xb, (int)T, (int)H,
                                   gamma, beta, eps, bits);
    }
    const float* xf = static_cast<const float*>(x);
    return gamma ? launch_smem(smooth_calib_kernel<float, true>, grid, block, smem, st, xf, (int)T, (int)H, gamma, beta,
                               eps, bits)
                 : launch_smem(smooth_calib_kernel<float, false>, grid, block, smem, st, xf, (int)T, (int)H, gamma, beta,
                               eps, bits);
}

int launch_smooth_weights(const float* W, int64_t N, int64_t K, const float* amax, float alpha, const float* gamma,
                          const float* beta, float* W_out, float* gamma_out, float* beta_out, float* s,
                          const DeviceInfo& di, cudaStream_t st) {
    int rc;
    // s holds the weight column maxima until the factor kernel replaces them
    if ((rc = cuda_status(cudaMemsetAsync(s, 0, (size_t)K * sizeof(float), st)))) return rc;
    const unsigned cblocks = (unsigned)((K + 255) / 256);
    if ((rc = launch(weight_col_absmax_kernel, dim3((unsigned)((K / 4 + 255) / 256), (unsigned)((N + kColRows - 1) / kColRows)),
                     dim3(256), st, W, N, K, reinterpret_cast<uint32_t*>(s))))
        return rc;
    if ((rc = launch(smooth_factor_kernel, dim3(cblocks), dim3(256), st, amax, s, K, (double)alpha, gamma, beta,
                     gamma_out, beta_out)))
        return rc;
    const int64_t n4 = N * K / 4;
    const int64_t want = (n4 + 255) / 256;
    const unsigned grid = (unsigned)(want < (int64_t)di.sm_count * 8 ? want : (int64_t)di.sm_count * 8);
    return launch(smooth_fold_kernel, dim3(grid), dim3(256), st, W, N, K, (const float*)s, W_out);
}

}  // namespace zq
