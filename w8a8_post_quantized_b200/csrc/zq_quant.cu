// zq_quant.cu -- memory-bound quantizer kernels for sm_100a:
//   * group-wise weight quantization (offline),
//   * fused LayerNorm + per-token quantization,
//   * fused (bias +) GeLU + per-token quantization,
//   * per-token requantization of an fp32 GEMM output with a known row absmax.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (group-wise weights, token-wise
// activations, the fused "LN/GeLU + Quantize" kernel) and
// "探秘Transformer系列之（36）— 大模型量化方案" §1.1.2 (absmax rule, [-127, 127])
// and §1.2.2 (dynamic per-token scales fused with the preceding LayerNorm).
//
// Row kernels keep the whole row in registers: the row is split into
// 16-element chunks (32 bytes of bf16 or 64 bytes of fp32 read with 16-byte
// loads, 16 int8 codes written with one 16-byte store); RT threads own a row
// and each holds VPT chunks.  Reductions (sum, sum of squares, absmax) use
// warp shuffles, then shared memory across the RT/32 warps of a row.  Each
// input byte is read from HBM once and each code written once.
#include "zq_internal.cuh"

namespace zq {
namespace {

// ------------------------------------------------------------ chunk loads

template <typename Tin>
struct Chunk;

template <>
struct Chunk<float> {
    static __device__ __forceinline__ void load(const float* p, float (&v)[16]) {
        const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float4 a = __ldcs(p4 + i);
            v[4 * i + 0] = a.x;
            v[4 * i + 1] = a.y;
            v[4 * i + 2] = a.z;
            v[4 * i + 3] = a.w;
        }
    }
};

template <>
struct Chunk<uint16_t> {  // bf16 bit patterns
    static __device__ __forceinline__ void load(const uint16_t* p, float (&v)[16]) {
        const uint4* p4 = reinterpret_cast<const uint4*>(p);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint4 a = __ldcs(p4 + i);
            const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                v[8 * i + 2 * j + 0] = bf16_lo(w[j]);
                v[8 * i + 2 * j + 1] = bf16_hi(w[j]);
            }
        }
    }
};

__device__ __forceinline__ void load16_f32_ldg(const float* p, float (&v)[16]) {
    const float4* p4 = reinterpret_cast<const float4*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float4 a = __ldg(p4 + i);
        v[4 * i + 0] = a.x;
        v[4 * i + 1] = a.y;
        v[4 * i + 2] = a.z;
        v[4 * i + 3] = a.w;
    }
}

__device__ __forceinline__ void store_codes16(int8_t* dst, const float (&y)[16], float inv) {
    uint4 o;
    o.x = pack_i8x4(quant_code(y[0], inv), quant_code(y[1], inv), quant_code(y[2], inv),
                    quant_code(y[3], inv));
    o.y = pack_i8x4(quant_code(y[4], inv), quant_code(y[5], inv), quant_code(y[6], inv),
                    quant_code(y[7], inv));
    o.z = pack_i8x4(quant_code(y[8], inv), quant_code(y[9], inv), quant_code(y[10], inv),
                    quant_code(y[11], inv));
    o.w = pack_i8x4(quant_code(y[12], inv), quant_code(y[13], inv), quant_code(y[14], inv),
                    quant_code(y[15], inv));
    __stcs(reinterpret_cast<uint4*>(dst), o);
}

// ------------------------------------------------------- row reductions

template <int RT>
__device__ __forceinline__ float row_sum(float v, float* sbuf) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if constexpr (RT == 32) {
        return v;
    } else {
        const int w = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) sbuf[w] = v;
        __syncthreads();
        const int w0 = (threadIdx.x / RT) * (RT / 32);
        float t = 0.0f;
#pragma unroll
        for (int i = 0; i < RT / 32; ++i) t += sbuf[w0 + i];
        __syncthreads();
        return t;
    }
}

template <int RT>
__device__ __forceinline__ float row_max(float v, float* sbuf) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if constexpr (RT == 32) {
        return v;
    } else {
        const int w = threadIdx.x >> 5;
        if ((threadIdx.x & 31) == 0) sbuf[w] = v;
        __syncthreads();
        const int w0 = (threadIdx.x / RT) * (RT / 32);
        float t = 0.0f;
#pragma unroll
        for (int i = 0; i < RT / 32; ++i) t = fmaxf(t, sbuf[w0 + i]);
        __syncthreads();
        return t;
    }
}

template <int RT>
__host__ __device__ constexpr int block_threads() { return RT >= 256 ? RT : 256; }

// ------------------------------------------------- LayerNorm + quantize

template <typename Tin, int RT, int VPT>
__global__ void __launch_bounds__(block_threads<RT>())
ln_quant_kernel(const Tin* __restrict__ x, int64_t T, int H, const float* __restrict__ gamma,
                const float* __restrict__ beta, float eps, int8_t* __restrict__ q,
                float* __restrict__ s_tok) {
    constexpr int ROWS = block_threads<RT>() / RT;
    __shared__ float sbuf[block_threads<RT>() / 32];
    const int tid = threadIdx.x % RT;
    const int64_t row = (int64_t)blockIdx.x * ROWS + threadIdx.x / RT;
    const bool row_ok = row < T;
    const int nch = H >> 4;

    float v[VPT][16];
    bool ok[VPT];
    float sum = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c = i * RT + tid;
        ok[i] = row_ok && c < nch;
        if (ok[i]) {
            Chunk<Tin>::load(x + row * H + (int64_t)c * 16, v[i]);
#pragma unroll
            for (int j = 0; j < 16; ++j) sum += v[i][j];
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) v[i][j] = 0.0f;
        }
    }
    const float mean = __fdiv_rn(row_sum<RT>(sum, sbuf), (float)H);
    float ss = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (ok[i]) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float d = v[i][j] - mean;
                ss = fmaf(d, d, ss);
            }
        }
    }
    const float var = __fdiv_rn(row_sum<RT>(ss, sbuf), (float)H);
    const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(var + eps));

    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        if (ok[i]) {
            const int c = i * RT + tid;
            float g[16], b[16];
            load16_f32_ldg(gamma + c * 16, g);
            load16_f32_ldg(beta + c * 16, b);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const float yv = fmaf((v[i][j] - mean) * rstd, g[j], b[j]);
                v[i][j] = yv;
                amax = fmaxf(amax, fabsf(yv));
            }
        }
    }
    amax = row_max<RT>(amax, sbuf);
    float scale, inv;
    absmax_scales(amax, scale, inv);
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        if (ok[i]) store_codes16(q + row * H + (int64_t)(i * RT + tid) * 16, v[i], inv);
    if (row_ok && tid == 0) s_tok[row] = scale;
}

// ---------------------------------------- (bias +) activation + quantize

template <typename Tin, int RT, int VPT>
__global__ void __launch_bounds__(block_threads<RT>())
act_quant_kernel(const Tin* __restrict__ x, int64_t T, int H, const float* __restrict__ bias,
                 int act, int8_t* __restrict__ q, float* __restrict__ s_tok) {
    constexpr int ROWS = block_threads<RT>() / RT;
    __shared__ float sbuf[block_threads<RT>() / 32];
    const int tid = threadIdx.x % RT;
    const int64_t row = (int64_t)blockIdx.x * ROWS + threadIdx.x / RT;
    const bool row_ok = row < T;
    const int nch = H >> 4;

    float v[VPT][16];
    bool ok[VPT];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
        const int c = i * RT + tid;
        ok[i] = row_ok && c < nch;
        if (ok[i]) {
            Chunk<Tin>::load(x + row * H + (int64_t)c * 16, v[i]);
            if (bias) {
                float b[16];
                load16_f32_ldg(bias + c * 16, b);
#pragma unroll
                for (int j = 0; j < 16; ++j) v[i][j] = __fadd_rn(v[i][j], b[j]);
            }
            if (act == ZQ_ACT_GELU) {
#pragma unroll
                for (int j = 0; j < 16; ++j) v[i][j] = gelu_f(v[i][j]);
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(v[i][j]));
        }
    }
    amax = row_max<RT>(amax, sbuf);
    float scale, inv;
    absmax_scales(amax, scale, inv);
#pragma unroll
    for (int i = 0; i < VPT; ++i)
        if (ok[i]) store_codes16(q + row * H + (int64_t)(i * RT + tid) * 16, v[i], inv);
    if (row_ok && tid == 0) s_tok[row] = scale;
}

// ------------------------------------------------ requantize GEMM output

// h fp32 [T, N], amax_bits[t] = bit pattern of the row's absmax (non-negative
// floats order like their bit patterns).  One 16-element chunk per thread
// iteration; N % 16 == 0 so a chunk never straddles rows.
__global__ void __launch_bounds__(256)
requant_rows_kernel(const float* __restrict__ h, int64_t n_chunks, int64_t chunks_per_row,
                    const uint32_t* __restrict__ amax_bits, int8_t* __restrict__ q,
                    float* __restrict__ s_tok) {
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n_chunks;
         c += (int64_t)gridDim.x * blockDim.x) {
        const int64_t row = c / chunks_per_row;
        const float amax = __uint_as_float(__ldg(amax_bits + row));
        float scale, inv;
        absmax_scales(amax, scale, inv);
        float v[16];
        Chunk<float>::load(h + c * 16, v);
        store_codes16(q + c * 16, v, inv);
        if (c - row * chunks_per_row == 0) s_tok[row] = scale;
    }
}

// ------------------------------------------------- weight quantization

// Pass 1: absmax of each group (G*K contiguous floats) into amax_bits[g].
// Block b works on group b / per_group, slice b % per_group.
__global__ void __launch_bounds__(256)
wq_absmax_kernel(const float* __restrict__ W, int64_t group_vec4, int per_group,
                 uint32_t* __restrict__ amax_bits) {
    __shared__ float sbuf[8];
    const int64_t g = blockIdx.x / per_group;
    const int slice = blockIdx.x % per_group;
    const float4* p = reinterpret_cast<const float4*>(W) + g * group_vec4;
    float m = 0.0f;
    for (int64_t i = (int64_t)slice * blockDim.x + threadIdx.x; i < group_vec4;
         i += (int64_t)per_group * blockDim.x) {
        const float4 a = __ldcs(p + i);
        m = fmaxf(m, fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(a.z), fabsf(a.w))));
    }
    m = row_max<256>(m, sbuf);
    if (threadIdx.x == 0) atomicMax(amax_bits + g, __float_as_uint(m));
}

// Pass 2: codes.  One 16-element chunk per thread iteration; K % 16 == 0.
__global__ void __launch_bounds__(256)
wq_quant_kernel(const float* __restrict__ W, int64_t n_chunks, int64_t chunks_per_group,
                const uint32_t* __restrict__ amax_bits, int8_t* __restrict__ Wq) {
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n_chunks;
         c += (int64_t)gridDim.x * blockDim.x) {
        const float amax = __uint_as_float(__ldg(amax_bits + c / chunks_per_group));
        float scale, inv;
        absmax_scales(amax, scale, inv);
        float v[16];
        Chunk<float>::load(W + c * 16, v);
        store_codes16(Wq + c * 16, v, inv);
    }
}

// Pass 3: the group scale replaces the absmax bits in place.
__global__ void wq_finalize_kernel(float* __restrict__ s_grp, int64_t n_groups) {
    const int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (g < n_groups) {
        float scale, inv;
        absmax_scales(s_grp[g], scale, inv);
        s_grp[g] = scale;
    }
}

// ------------------------------------------------------------ dispatch

template <typename Tin>
using RowKernel = void (*)(const Tin*, int64_t, int, const float*, const float*, float, int8_t*,
                           float*);
template <typename Tin>
using ActKernel = void (*)(const Tin*, int64_t, int, const float*, int, int8_t*, float*);

// Smallest RT in {32, ..., 1024} with RT*4 >= chunks; VPT = ceil(chunks/RT).
static void pick_row_shape(int H, int& RT, int& VPT) {
    const int chunks = H / 16;
    RT = 32;
    while (RT * 4 < chunks) RT *= 2;
    VPT = (chunks + RT - 1) / RT;
}

#define ZQ_ROW_TABLE(KERNEL, TIN)                                                          \
    {                                                                                      \
        {KERNEL<TIN, 32, 1>, KERNEL<TIN, 32, 2>, KERNEL<TIN, 32, 3>, KERNEL<TIN, 32, 4>},  \
            {KERNEL<TIN, 64, 1>, KERNEL<TIN, 64, 2>, KERNEL<TIN, 64, 3>,                   \
             KERNEL<TIN, 64, 4>},                                                          \
            {KERNEL<TIN, 128, 1>, KERNEL<TIN, 128, 2>, KERNEL<TIN, 128, 3>,                \
             KERNEL<TIN, 128, 4>},                                                         \
            {KERNEL<TIN, 256, 1>, KERNEL<TIN, 256, 2>, KERNEL<TIN, 256, 3>,                \
             KERNEL<TIN, 256, 4>},                                                         \
            {KERNEL<TIN, 512, 1>, KERNEL<TIN, 512, 2>, KERNEL<TIN, 512, 3>,                \
             KERNEL<TIN, 512, 4>},                                                         \
        {                                                                                  \
            KERNEL<TIN, 1024, 1>, KERNEL<TIN, 1024, 2>, KERNEL<TIN, 1024, 3>,              \
                KERNEL<TIN, 1024, 4>                                                       \
        }                                                                                  \
    }

static int log2_rt_index(int RT) {
    int i = 0;
    while ((32 << i) < RT) ++i;
    return i;
}

template <typename Tin>
static int launch_ln_typed(const Tin* x, int64_t T, int64_t H, const float* gamma,
                           const float* beta, float eps, int8_t* q, float* s_tok, cudaStream_t st) {
    static const RowKernel<Tin> table[6][4] = ZQ_ROW_TABLE(ln_quant_kernel, Tin);
    int RT, VPT;
    pick_row_shape((int)H, RT, VPT);
    const int threads = RT >= 256 ? RT : 256;
    const int rows = threads / RT;
    const int64_t blocks = (T + rows - 1) / rows;
    count_launch();
    table[log2_rt_index(RT)][VPT - 1]<<<(unsigned)blocks, threads, 0, st>>>(
        x, T, (int)H, gamma, beta, eps, q, s_tok);
    return cuda_status(cudaGetLastError());
}

template <typename Tin>
static int launch_act_typed(const Tin* x, int64_t T, int64_t H, const float* bias, int act,
                            int8_t* q, float* s_tok, cudaStream_t st) {
    static const ActKernel<Tin> table[6][4] = ZQ_ROW_TABLE(act_quant_kernel, Tin);
    int RT, VPT;
    pick_row_shape((int)H, RT, VPT);
    const int threads = RT >= 256 ? RT : 256;
    const int rows = threads / RT;
    const int64_t blocks = (T + rows - 1) / rows;
    count_launch();
    table[log2_rt_index(RT)][VPT - 1]<<<(unsigned)blocks, threads, 0, st>>>(x, T, (int)H, bias,
                                                                            act, q, s_tok);
    return cuda_status(cudaGetLastError());
}

}  // namespace

int launch_ln_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* gamma,
                    const float* beta, float eps, int8_t* q, float* s_tok, const DeviceInfo& di,
                    cudaStream_t st) {
    // pipelined kernel first; rows too long for it use the register kernel below
    const int rc = launch_rowq_pipe(x, x_dtype, T, H, true, gamma, beta, eps, nullptr, 0, q, s_tok, di, st);
    if (rc != ZQ_ERR_SHAPE) return rc;
    if (x_dtype == ZQ_BF16)
        return launch_ln_typed(static_cast<const uint16_t*>(x), T, H, gamma, beta, eps, q, s_tok, st);
    return launch_ln_typed(static_cast<const float*>(x), T, H, gamma, beta, eps, q, s_tok, st);
}

int launch_act_quant(const void* x, int x_dtype, int64_t T, int64_t H, const float* bias, int act,
                     int8_t* q, float* s_tok, const DeviceInfo& di, cudaStream_t st) {
    const int rc = launch_rowq_pipe(x, x_dtype, T, H, false, nullptr, nullptr, 0.f, bias, act, q, s_tok, di, st);
    if (rc != ZQ_ERR_SHAPE) return rc;
    if (x_dtype == ZQ_BF16)
        return launch_act_typed(static_cast<const uint16_t*>(x), T, H, bias, act, q, s_tok, st);
    return launch_act_typed(static_cast<const float*>(x), T, H, bias, act, q, s_tok, st);
}

int launch_requant_rows(const float* h, int64_t T, int64_t N, const uint32_t* amax_bits, int8_t* q,
                        float* s_tok, const DeviceInfo& di, cudaStream_t st) {
    const int64_t n_chunks = T * N / 16;
    int64_t blocks = (n_chunks + 255) / 256;
    const int64_t cap = (int64_t)di.sm_count * 8;
    if (blocks > cap) blocks = cap;
    count_launch();
    requant_rows_kernel<<<(unsigned)blocks, 256, 0, st>>>(h, n_chunks, N / 16, amax_bits, q, s_tok);
    return cuda_status(cudaGetLastError());
}

int launch_quantize_weights(const float* W, int64_t N, int64_t K, int64_t G, int8_t* Wq,
                            float* s_grp, const DeviceInfo& di, cudaStream_t st) {
    const int64_t n_groups = N / G;
    uint32_t* amax_bits = reinterpret_cast<uint32_t*>(s_grp);  // scratch until pass 3
    int rc = cuda_status(cudaMemsetAsync(amax_bits, 0, n_groups * sizeof(float), st));
    if (rc) return rc;
    const int64_t group_vec4 = G * K / 4;
    // enough blocks in total to cover every SM several times
    int64_t per_group = (4 * (int64_t)di.sm_count + n_groups - 1) / n_groups;
    const int64_t max_useful = (group_vec4 + 256 * 4 - 1) / (256 * 4);
    if (per_group > max_useful) per_group = max_useful;
    if (per_group < 1) per_group = 1;
    if (per_group > 4096) per_group = 4096;
    count_launch();
    wq_absmax_kernel<<<(unsigned)(per_group * n_groups), 256, 0, st>>>(W, group_vec4,
                                                                       (int)per_group, amax_bits);
    if ((rc = cuda_status(cudaGetLastError()))) return rc;
    const int64_t n_chunks = N * K / 16;
    int64_t blocks = (n_chunks + 255) / 256;
    const int64_t cap = (int64_t)di.sm_count * 8;
    if (blocks > cap) blocks = cap;
    count_launch();
    wq_quant_kernel<<<(unsigned)blocks, 256, 0, st>>>(W, n_chunks, G * K / 16, amax_bits, Wq);
    if ((rc = cuda_status(cudaGetLastError()))) return rc;
    count_launch();
    wq_finalize_kernel<<<(unsigned)((n_groups + 255) / 256), 256, 0, st>>>(s_grp, n_groups);
    return cuda_status(cudaGetLastError());
}

}  // namespace zq
