// zq_gemm_sk.cu -- W8A8 linear for few tokens (at most 64: decode), with the
// work divided evenly over all SMs ("stream-K").
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (the fused "GEMM + DeQuantize"
// kernel) and "探秘Transformer系列之（36）— 大模型量化方案" §1.2.2 (INT32
// accumulation scaled by the activation and weight scales before the write).
//
// With few tokens the weights dominate the traffic, so the operand roles are
// swapped: 128 weight rows fill the MMA's M side and the tokens (rounded up
// to BN = 16, 32 or 64) are its N side.  The (weight tile, k-block)
// iterations, m_tiles * ceil(K/128) of them in tile order, are cut into equal
// contiguous ranges, one per persistent CTA (one CTA per SM), so every SM
// streams the same number of weight bytes whatever the tile count.  A range
// boundary inside a tile splits it:
//   - the CTA whose range holds the tile's FIRST k-block finalizes the tile;
//     that piece is the last one of its range;
//   - every other piece of the tile starts a later CTA's range: that CTA
//     computes it first, writes its int32 partial accumulators to the
//     workspace and raises its flag (release);
//   - the finalizer, at the end of its range, waits (acquire, bounded) for
//     the flags of the CTAs that hold the rest of the tile, adds their
//     partials to its own (exact int32 sums) and runs the epilogue.
// Contributors never wait on anything before publishing, so every wait ends
// once all CTAs are resident: the grid has at most one CTA per SM (one fits,
// by its shared memory and TMEM), and every CTA signals dependent launches
// right after its prologue, so a later kernel cannot take an SM before all
// of them are running.  The flags are zeroed by a small kernel launched just
// before.  Every wait is bounded.
//
// The route is taken when every range holds at least a whole tile's worth of
// iterations (at least as many weight tiles as SMs).  With fewer tiles, some
// range lies inside one tile: its piece ends with the range while the
// tile's finalizer waits for it, and the exchange through global memory
// (about 2 us measured) lands on the critical path; the split-K clusters,
// which exchange partials through distributed shared memory, do better there.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int BM = 128;
constexpr int BK = 128;
constexpr int UMMA_K = 32;
constexpr int EW = 4;                         // epilogue warps: one per TMEM lane quarter
constexpr int kThreads = 64 + 32 * EW;
constexpr int kEpiThreads = 32 * EW;
constexpr int A_STAGE = BM * BK;              // weight stage: 128 rows x 128 bytes
constexpr int kMaxBN = 64;
enum { SK_F32 = 0, SK_BF16 = 1, SK_I32 = 2 };

enum {
    SITE_SK_P_EMPTY = 0x701,
    SITE_SK_P_DRAIN = 0x702,
    SITE_SK_M_TEMPTY = 0x703,
    SITE_SK_M_FULL = 0x704,
    SITE_SK_M_DRAIN = 0x705,
    SITE_SK_E_TFULL = 0x706,
    SITE_SK_E_PART = 0x707,
};

struct SkParams {
    int M;            // weight rows (output features)
    int Nt;           // tokens
    int K, G;
    int kb_per_tile;  // ceil(K / 128)
    int total;        // m_tiles * kb_per_tile iterations
    int per_cta;      // iterations per CTA (the last CTA may have fewer)
    const float* s_tok;
    const float* s_grp;
    const float* bias;  // may be null
    void* y;            // [Nt, M]
    int act;
    int32_t* part;      // [gridDim][kMaxBN columns][BM rows] partial accumulators
    uint32_t* flag;     // [gridDim], zero on entry
    int* status;
};

template <int BN>
__host__ __device__ constexpr uint32_t sk_tmem_cols() {
    return 2 * BN <= 32 ? 32 : 2 * BN <= 64 ? 64 : 128;
}

template <int BN, int STAGES>
__host__ __device__ constexpr size_t sk_smem() {
    // alignment slack + operand ring + barriers/flags (256) + token scales
    return 1024 + (size_t)STAGES * (A_STAGE + BN * BK) + 256 + kMaxBN * 4;
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// The pieces of this CTA's iteration range, in order: (tile, first k-block,
// end k-block).
struct Piece {
    int t, kb_lo, kb_hi;
};
__device__ __forceinline__ Piece piece_at(int it, int it_end, int KB) {
    Piece pc;
    pc.t = it / KB;
    pc.kb_lo = it - pc.t * KB;
    pc.kb_hi = min(KB, pc.kb_lo + (it_end - it));
    return pc;
}

template <int BN, int STAGES, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_decode_sk_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                      const SkParams p) {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= kMaxBN, "tokens as MMA N: 16..64");
    static_assert(8 * (2 * STAGES + 5) + 8 <= 256, "barriers and flags fit their 256 bytes");
    constexpr int B_STAGE = BN * BK;
    constexpr uint32_t IDESC = idesc_i8(BM, BN);
    constexpr uint32_t TMEM_COLS = sk_tmem_cols<BN>();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * A_STAGE;
    const uint32_t sBar = sB + STAGES * B_STAGE;
    uint8_t* gBar = gbase + (sBar - base);
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain
    auto bar_full = [&](int s) { return sBar + 8u * s; };
    auto bar_empty = [&](int s) { return sBar + 8u * (STAGES + s); };
    auto bar_tfull = [&](int b) { return sBar + 8u * (2 * STAGES + b); };
    auto bar_tempty = [&](int b) { return sBar + 8u * (2 * STAGES + 2 + b); };
    const uint32_t bar_drain = sBar + 8u * (2 * STAGES + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* tok_scale = reinterpret_cast<float*>(gBar + 256);  // [kMaxBN]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int KB = p.kb_per_tile;
    const int it0 = (int)blockIdx.x * p.per_cta;
    const int it1 = min(it0 + p.per_cta, p.total);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull(b), 1);
            mbar_init(bar_tempty(b), EW);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_proxy_async_smem();
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The weights are never written by a kernel that lets its successor start
    // early, so the producer streams the first ring of weight tiles before
    // waiting for the previous grid; every role waits before it touches the
    // tokens, the token scales, the workspace or the output.
    griddep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            const int n = it1 - it0;
            const int npre = min(STAGES, max(n, 0));
            for (int j = 0; j < npre; ++j) {
                const int it = it0 + j;
                const int t = it / KB;
                mbar_arrive_expect_tx(bar_full(j), A_STAGE + B_STAGE);
                tma_load_2d(sA + j * A_STAGE, &tmW, bar_full(j), (it - t * KB) * BK, t * BM);
            }
            griddep_wait();
            int j = 0;
            for (; j < n; ++j) {
                const int it = it0 + j;
                const int t = it / KB;
                const int kb = it - t * KB;
                const int s = j % STAGES;
                const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                if (j >= npre) {
                    if (!mbar_wait(bar_empty(s), ph ^ 1u, abort_flag, p.status, SITE_SK_P_EMPTY)) break;
                    mbar_arrive_expect_tx(bar_full(s), A_STAGE + B_STAGE);
                    tma_load_2d(sA + s * A_STAGE, &tmW, bar_full(s), kb * BK, t * BM);
                }
                tma_load_2d(sB + s * B_STAGE, &tmX, bar_full(s), kb * BK, 0);
            }
            // every copy this thread issued lands before the CTA can exit
            const int issued = max(j, npre);
            for (int jj = max(0, issued - STAGES); jj < issued; ++jj)
                mbar_wait(bar_full(jj % STAGES), (uint32_t)(jj / STAGES) & 1u, nullptr, p.status, SITE_SK_P_DRAIN);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            int j = 0;
            uint32_t u = 0;
            bool ok = true;
            for (int it = it0; ok && it < it1; ++u) {
                const Piece pc = piece_at(it, it1, KB);
                const int b = u & 1;
                if (!mbar_wait(bar_tempty(b), ((u >> 1) & 1u) ^ 1u, abort_flag, p.status, SITE_SK_M_TEMPTY)) break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                for (int kb = pc.kb_lo; kb < pc.kb_hi; ++kb, ++j) {
                    const int s = j % STAGES;
                    const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                    if (!mbar_wait(bar_full(s), ph, abort_flag, p.status, SITE_SK_M_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw128(sA + s * A_STAGE);
                    const uint64_t db = sdesc_k_sw128(sB + s * B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        mma_i8(d_tmem, da + 2u * k, db + 2u * k, IDESC, (kb > pc.kb_lo || k > 0) ? 1u : 0u);
                    mma_commit(bar_empty(s));
                }
                if (ok) mma_commit(bar_tfull(b));
                it += pc.kb_hi - pc.kb_lo;
            }
            mma_commit(bar_drain);
            mbar_wait(bar_drain, 0u, nullptr, p.status, SITE_SK_M_DRAIN);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        griddep_wait();  // token scales and the zeroed flags belong to earlier grids
        const int quarter = warp & 3;        // TMEM lanes 32*quarter .. +31
        const int r = quarter * 32 + lane;   // weight row of the tile owned by this thread
        const int et = threadIdx.x - 64;
        for (int i = et; i < kMaxBN; i += kEpiThreads) tok_scale[i] = i < p.Nt ? __ldg(p.s_tok + i) : 0.0f;
        named_bar_sync(1, kEpiThreads);
        const bool gelu = p.act == ZQ_ACT_GELU;
        uint32_t u = 0;
        for (int it = it0; it < it1; ++u) {
            const Piece pc = piece_at(it, it1, KB);
            it += pc.kb_hi - pc.kb_lo;
            const int b = u & 1;
            // the factors of this thread's weight row, loaded before the wait
            const int gm = pc.t * BM + r;
            float row_scale = 0.0f, row_bias = 0.0f;
            if (EPI != SK_I32 && pc.kb_lo == 0 && gm < p.M) {
                row_scale = __ldg(p.s_grp + gm / p.G);
                row_bias = p.bias ? __ldg(p.bias + gm) : 0.0f;
            }
            const bool got = mbar_wait(bar_tfull(b), (u >> 1) & 1u, abort_flag, p.status, SITE_SK_E_TFULL);
            if (!named_bar_and(1, kEpiThreads, got)) break;
            tc_fence_after();
            // this thread's row of the piece's accumulator, into registers;
            // the accumulator is free again
            uint32_t v[BN];
            const uint32_t t_row = tmem_base + (uint32_t)(b * BN) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
            for (int c = 0; c < BN / 16; ++c) {
                uint32_t w16[16];
                tmem_ld_32x32b_x16(t_row + c * 16, w16);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) v[c * 16 + i] = w16[i];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty(b));
            // partials are stored column-major per CTA ([kMaxBN][BM] int32),
            // so a warp's accesses to one column are 128 contiguous bytes
            if (pc.kb_lo > 0) {
                // a later piece of the tile: publish the partial for its finalizer
                int32_t* my_part = p.part + (size_t)blockIdx.x * BM * kMaxBN + r;
#pragma unroll
                for (int j = 0; j < BN; ++j) my_part[j * BM] = (int32_t)v[j];
                __threadfence();
                named_bar_sync(1, kEpiThreads);
                if (et == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.flag + blockIdx.x), "r"(1u) : "memory");
                continue;
            }
            if (pc.kb_hi < KB) {
                // the tile's first piece: add the partials of the CTAs that hold
                // the rest of it (ranges start in order, so they are the next ones)
                const int last = (pc.t * KB + KB - 1) / p.per_cta;
                bool ok = true;
                for (int c2 = (int)blockIdx.x + 1; c2 <= last; ++c2) {
                    if (et == 0) {
                        const uint64_t t0 = globaltimer_ns();
                        while (ld_acquire_u32(p.flag + c2) == 0u) {
                            if (*abort_flag || globaltimer_ns() - t0 > kWaitLimitNs) {
                                atomicCAS(p.status, 0, SITE_SK_E_PART);
                                *abort_flag = 1;
                                ok = false;
                                break;
                            }
                            __nanosleep(64);
                        }
                    }
                    if (!named_bar_and(1, kEpiThreads, ok)) {
                        ok = false;
                        break;
                    }
                    const int32_t* src = p.part + (size_t)c2 * BM * kMaxBN + r;
#pragma unroll
                    for (int j = 0; j < BN; ++j) {
                        uint32_t q;
                        asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(q) : "l"(src + j * BM) : "memory");
                        v[j] += q;
                    }
                }
                if (!ok) break;
            }
            // epilogue of the whole tile: weight row gm, tokens 0 .. Nt-1
            if (gm < p.M) {
#pragma unroll
                for (int j = 0; j < BN; ++j) {
                    if (j >= p.Nt) break;
                    const int64_t off = (int64_t)j * p.M + gm;
                    if constexpr (EPI == SK_I32) {
                        static_cast<int32_t*>(p.y)[off] = (int32_t)v[j];
                    } else {
                        float t = fmaf(row_scale * tok_scale[j], (float)(int)v[j], row_bias);
                        if (gelu) t = gelu_f(t);
                        if constexpr (EPI == SK_BF16) static_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(t);
                        else static_cast<float*>(p.y)[off] = t;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

constexpr int kMaxDevices = 64;
// ring depth: 8 stages measured faster on the 16-token decode layer than 6
// (3% slower) and than 12, the most that fits (5% slower)
template <int BN>
constexpr int stages_sk() { return 8; }

template <int BN, int EPI>
int sk_launch(const CUtensorMap& tw, const CUtensorMap& tx, const SkParams& p, int grid, cudaStream_t st) {
    constexpr int kStagesSK = stages_sk<BN>();
    constexpr size_t kSmem = sk_smem<BN, kStagesSK>();
    static_assert(kSmem <= 232448, "shared memory budget");
    auto kern = w8a8_decode_sk_kernel<BN, kStagesSK, EPI>;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    {
        static bool attr_set[kMaxDevices] = {};
        std::lock_guard<std::mutex> lk(launch_cache_mutex());
        if (!attr_set[dev]) {
            int rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
            if (rc) return rc;
            attr_set[dev] = true;
        }
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, tw, tx, p));
}

template <int BN>
int sk_launch_epi(int epi, const CUtensorMap& tw, const CUtensorMap& tx, const SkParams& p, int grid,
                  cudaStream_t st) {
    if (epi == SK_F32) return sk_launch<BN, SK_F32>(tw, tx, p, grid, st);
    if (epi == SK_BF16) return sk_launch<BN, SK_BF16>(tw, tx, p, grid, st);
    return sk_launch<BN, SK_I32>(tw, tx, p, grid, st);
}

// Zeroes the partial-ready flags; lets the linear launch at once and waits for
// the previous grid before writing (an earlier call may still read them).
__global__ void zero_flags_kernel(uint32_t* __restrict__ w, int n) {
    griddep_launch_dependents();
    griddep_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) w[i] = 0u;
}

int launch_zero_flags(uint32_t* flag, int n, cudaStream_t st) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, zero_flags_kernel, flag, n));
}

}  // namespace

bool decode_even_applies(int64_t T, int64_t K, int64_t N, int sms) {
    if (T > kMaxBN || sms <= 0) return false;
    const int64_t KB = (K + BK - 1) / BK;
    const int64_t total = ((N + BM - 1) / BM) * KB;
    if (total > (1ll << 30)) return false;
    const int mode = even_split_mode();
    if (mode == 1) return false;
    if (mode == 2) return true;
    // every range holds at least a whole tile's worth of iterations
    const int64_t per = (total + sms - 1) / sms;
    return per >= KB;
}

size_t decode_sk_ws_bytes(int sms) {
    if (sms <= 0) return 0;
    const size_t part = (size_t)sms * BM * kMaxBN * sizeof(int32_t);
    return part + ((size_t)sms * sizeof(uint32_t) + 255) / 256 * 256;
}

int launch_w8a8_decode_sk(const LinearArgs& a, void* ws, size_t ws_bytes, const DeviceInfo& di, cudaStream_t st) {
    if (a.T > kMaxBN) return ZQ_ERR_SHAPE;
    int epi;
    switch (a.out_kind) {
        case ZQ_OUT_F32: epi = SK_F32; break;
        case ZQ_OUT_BF16: epi = SK_BF16; break;
        case ZQ_OUT_I32_RAW: epi = SK_I32; break;
        default: return ZQ_ERR_SHAPE;
    }
    const size_t need = decode_sk_ws_bytes(di.sm_count);
    if (!ws || ws_bytes < need) return ZQ_ERR_WORKSPACE;
    const int64_t KB = (a.K + BK - 1) / BK;
    const int64_t m_tiles = (a.N + BM - 1) / BM;
    const int64_t total = m_tiles * KB;
    if (total > (1ll << 30)) return ZQ_ERR_SHAPE;
    const int64_t per_cta = (total + di.sm_count - 1) / di.sm_count;
    const int grid = (int)((total + per_cta - 1) / per_cta);
    int32_t* part = static_cast<int32_t*>(ws);
    uint32_t* flag = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + (size_t)di.sm_count * BM * kMaxBN * 4);
    int rc;
    if ((rc = launch_zero_flags(flag, grid, st))) return rc;
    const int bn = a.T <= 16 ? 16 : a.T <= 32 ? 32 : 64;
    CUtensorMap tw, tx;
    if ((rc = make_tmap_i8(&tw, a.Wq, a.N, a.K, BM))) return rc;
    if ((rc = make_tmap_i8(&tx, a.xq, a.T, a.K, bn))) return rc;
    SkParams p{};
    p.M = (int)a.N;
    p.Nt = (int)a.T;
    p.K = (int)a.K;
    p.G = (int)a.G;
    p.kb_per_tile = (int)KB;
    p.total = (int)total;
    p.per_cta = (int)per_cta;
    p.s_tok = a.s_tok;
    p.s_grp = a.s_grp;
    p.bias = a.bias;
    p.y = a.y;
    p.act = a.act;
    p.part = part;
    p.flag = flag;
    p.status = di.status_word;
    if (bn == 16) return sk_launch_epi<16>(epi, tw, tx, p, grid, st);
    if (bn == 32) return sk_launch_epi<32>(epi, tw, tx, p, grid, st);
    return sk_launch_epi<64>(epi, tw, tx, p, grid, st);
}

}  // namespace zq
