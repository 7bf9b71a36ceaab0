// zq_gemm_greq.cu -- W8A8 linear whose epilogue requantizes each output row
// per token for the next layer, for rows of any width: one persistent kernel,
// no fp32 intermediate in HBM.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (the fused "GEMM + DeQuantize"
// kernel; token-wise quantization fused with the op that produces the
// activations) and "探秘Transformer系列之（36）— 大模型量化方案" §1.2.2 (INT32
// accumulators scaled by the weight and activation scales before the next
// op; one dynamic scale per token, over the whole row).
//
// The per-token scale needs the absmax of a whole output row, which spans
// n_t = N / 256 accumulator tiles computed by different CTAs.  Tiles are
// numbered row block first (tile t = row block t / n_t, column tile t % n_t)
// and CTA c of the P co-resident CTAs takes tiles c, c + P, c + 2P, ...  For
// each tile the epilogue
//   pass 1  dequantizes, adds bias, applies GeLU (packed fp32 pairs) and keeps
//           the fp32 results of its row slice in registers, so the TMEM
//           accumulator is released at once and the next tile's MMA proceeds;
//   publish combines the row maxima of the CTA's four column slices, raises
//           the row's absmax word in global memory (atomicMax on the bit
//           pattern: non-negative floats order like their bits) and counts
//           the tile on its row block's arrival counter (release);
//   wait    until the counter reaches n_t (acquire), then reads the row absmax;
//   pass 2  writes the int8 codes, scale = absmax/127, code =
//           rint(fl(h * fl(127/absmax))), with TMA stores.
// Progress: a tile's pass 2 waits for the tiles of its row block, whose own
// epilogues wait at most for the pass 2 of the tile P places earlier on the
// same CTA.  With n_t <= P every wait therefore points to a lower tile index,
// so all waits end once every CTA is resident (grid <= SMs, one CTA per SM).
// The absmax words and counters live in the caller's workspace and are
// zeroed by a small kernel launched just before this one.  Every wait is
// bounded.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int UMMA_K = 32;
constexpr int EW = 16;                 // epilogue warps: 4 TMEM lane quarters x 4 column slices
constexpr int kThreads = 64 + 32 * EW;
constexpr int kEpiThreads = 32 * EW;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr uint32_t kTmemCols = 512;    // two 256-column accumulators
constexpr int kStages = 4;

enum {
    SITE_P_EMPTY = 0x601,
    SITE_P_DRAIN = 0x602,
    SITE_M_TEMPTY = 0x603,
    SITE_M_FULL = 0x604,
    SITE_M_DRAIN = 0x605,
    SITE_E_TFULL = 0x606,
    SITE_E_ROWS = 0x607,
};

struct Params {
    int M, N, K, G;
    int n_t, m_tiles;
    const float* s_tok;
    const float* s_grp;
    const float* bias;       // may be null
    float* s_tok_out;        // [M]
    uint32_t* amax;          // [M] absmax bit patterns, zero on entry
    uint32_t* count;         // [m_tiles] tiles published per row block, zero on entry
    int act;
    int* status;
};

__host__ __device__ constexpr size_t smem_bytes() {
    // 1024 alignment slack + operand ring + one 32x32 int8 staging box per
    // epilogue warp + barriers/flags (256) + row partials of the slices [4][BM]
    return 1024 + (size_t)kStages * (A_STAGE + B_STAGE) + EW * 32 * 32 + 256 + 4 * BM * 4;
}

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Bounded wait until *cnt >= target (acquire at GPU scope).  Gives up when
// the CTA's abort flag is raised or after kWaitLimitNs (records `site`).
__device__ bool wait_count(const uint32_t* cnt, uint32_t target, volatile int* abort_flag, int* status, int site) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t n = 1;; ++n) {
        __nanosleep(64);
        if (ld_acquire_gpu(cnt) >= target) return true;
        if ((n & 15u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                atomicCAS(status, 0, site);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
w8a8_requant_grid_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmY, const Params p) {
    constexpr uint32_t IDESC = idesc_i8(BM, BN);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + kStages * A_STAGE;
    const uint32_t sStg = sB + kStages * B_STAGE;   // [EW][32 rows][32 B], 1024-aligned
    const uint32_t sBar = sStg + EW * 32 * 32;
    uint8_t* gBar = gbase + (sBar - base);
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain
    auto bar_full = [&](int s) { return sBar + 8u * s; };
    auto bar_empty = [&](int s) { return sBar + 8u * (kStages + s); };
    auto bar_tfull = [&](int b) { return sBar + 8u * (2 * kStages + b); };
    auto bar_tempty = [&](int b) { return sBar + 8u * (2 * kStages + 2 + b); };
    const uint32_t bar_drain = sBar + 8u * (2 * kStages + 4);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * kStages + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* slice_part = reinterpret_cast<float*>(gBar + 256);   // [4][BM]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.m_tiles * p.n_t;
    const int kblocks = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
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
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // The weights (codes, group scales, bias) are never written by a kernel
    // that lets its successor start early, so the producer streams the first
    // ring of weight tiles before waiting for the previous grid; every role
    // waits before it touches activations, the scratch words or outputs.
    griddep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t npre = 0;
            for (int t = blockIdx.x; npre < (uint32_t)kStages && t < num_tiles; t += gridDim.x) {
                const int nt = t % p.n_t;
                for (int kb = 0; kb < kblocks && npre < (uint32_t)kStages; ++kb, ++npre) {
                    mbar_arrive_expect_tx(bar_full((int)npre), A_STAGE + B_STAGE);
                    tma_load_2d(sB + npre * B_STAGE, &tmB, bar_full((int)npre), kb * BK, nt * BN);
                }
            }
            griddep_wait();
            uint32_t it = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x) {
                const int mt = t / p.n_t, nt = t % p.n_t;
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (it >= npre) {
                        if (!mbar_wait(bar_empty(s), ph ^ 1u, abort_flag, p.status, SITE_P_EMPTY)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_full(s), A_STAGE + B_STAGE);
                        tma_load_2d(sB + s * B_STAGE, &tmB, bar_full(s), kb * BK, nt * BN);
                    }
                    tma_load_2d(sA + s * A_STAGE, &tmA, bar_full(s), kb * BK, mt * BM);
                }
            }
            const uint32_t first = it > (uint32_t)kStages ? it - kStages : 0u;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(bar_full(j % kStages), (j / kStages) & 1u, nullptr, p.status, SITE_P_DRAIN);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < num_tiles; t += gridDim.x, ++lt) {
                const int b = lt & 1;
                if (!mbar_wait(bar_tempty(b), ((lt >> 1) & 1u) ^ 1u, abort_flag, p.status, SITE_M_TEMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                for (int kb = 0; kb < kblocks; ++kb, ++it) {
                    const int s = it % kStages;
                    const uint32_t ph = (it / kStages) & 1u;
                    if (!mbar_wait(bar_full(s), ph, abort_flag, p.status, SITE_M_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw128(sA + s * A_STAGE);
                    const uint64_t db = sdesc_k_sw128(sB + s * B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        mma_i8(d_tmem, da + 2u * k, db + 2u * k, IDESC, (kb | k) != 0 ? 1u : 0u);
                    mma_commit(bar_empty(s));
                }
                if (ok) mma_commit(bar_tfull(b));
            }
            mma_commit(bar_drain);
            mbar_wait(bar_drain, 0u, nullptr, p.status, SITE_M_DRAIN);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        griddep_wait();  // token scales, the zeroed scratch words and y belong to earlier grids
        constexpr int CW = 32;
        const int quarter = warp & 3;                  // TMEM lanes 32*quarter .. +31
        const int slice = (warp - 2) >> 2;             // columns 64*slice .. +63 of the tile
        const int r = quarter * 32 + lane;             // tile row owned by this thread
        const int et = threadIdx.x - 64;
        uint8_t* stg = gbase + (sStg - base) + (uint32_t)(warp - 2) * 32u * 32u;
        const uint32_t stg_s = smem_u32(stg);
        const bool gelu = p.act == ZQ_ACT_GELU;
        const bool uni = p.G % CW == 0;                // every 32-column chunk lies in one weight group
        // column factors of the next chunk (lane l: column l's group scale and
        // bias) and the next tile's token scale, loaded one step ahead
        float pa = 0.0f, pb = 0.0f, prs = 0.0f;
        auto fetch_cols = [&](int t, int c) {
            const int n = (t % p.n_t) * BN + slice * 64 + c * CW + lane;
            const bool in = n < p.N;
            pa = in ? __ldg(p.s_grp + n / p.G) : 0.0f;
            pb = (in && p.bias) ? __ldg(p.bias + n) : 0.0f;
        };
        auto fetch_row = [&](int t) {
            const int gm = (t / p.n_t) * BM + r;
            prs = gm < p.M ? __ldg(p.s_tok + gm) : 0.0f;
        };
        if ((int)blockIdx.x < num_tiles) {
            fetch_cols(blockIdx.x, 0);
            fetch_row(blockIdx.x);
        }
        uint32_t lt = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++lt) {
            const int mt = t / p.n_t, nt = t % p.n_t;
            const int b = lt & 1;
            const int gm = mt * BM + r;
            const bool row_ok = gm < p.M;
            const float row_scale = prs;
            if (t + (int)gridDim.x < num_tiles) fetch_row(t + gridDim.x);
            // pass 1: the two 32-column chunks of this thread's slice, kept as
            // packed fp32 pairs; the accumulator is released right after
            const bool got = __all_sync(0xFFFFFFFFu, mbar_wait(bar_tfull(b), (lt >> 1) & 1u, abort_flag, p.status,
                                                               SITE_E_TFULL));
            uint64_t h[2][16];
            float pmax = 0.0f;
            if (got) {
                tc_fence_after();
                const uint32_t t_row = tmem_base + (uint32_t)(b * BN + slice * 64) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const float ca = pa, cb = pb;
                    if (c == 0) fetch_cols(t, 1);
                    else if (t + (int)gridDim.x < num_tiles) fetch_cols(t + gridDim.x, 0);
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + c * CW, v);
                    tmem_ld_wait();
                    if (gelu) {
                        if (uni) dequant_chunk_lanes<true, true>(v, row_scale, ca, cb, h[c]);
                        else dequant_chunk_lanes<true, false>(v, row_scale, ca, cb, h[c]);
                    } else {
                        if (uni) dequant_chunk_lanes<false, true>(v, row_scale, ca, cb, h[c]);
                        else dequant_chunk_lanes<false, false>(v, row_scale, ca, cb, h[c]);
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        float t0, t1;
                        f2_unpack(h[c][i], t0, t1);
                        pmax = fmaxf(pmax, fmaxf(fabsf(t0), fabsf(t1)));   // columns past N add 0
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_tempty(b));
            }
            // publish: the row maxima of the four slices, one atomic per row,
            // then one arrival for the tile on its row block's counter
            slice_part[slice * BM + r] = pmax;
            if (!named_bar_and(1, kEpiThreads, got)) break;
            if (slice == 0) {
                if (row_ok) {
                    float m = slice_part[r];
#pragma unroll
                    for (int s = 1; s < 4; ++s) m = fmaxf(m, slice_part[s * BM + r]);
                    atomicMax(p.amax + gm, __float_as_uint(m));
                }
                __threadfence();                 // the row maxima before the arrival below
                named_bar_sync(2, 128);
                if (et == 0) {
                    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(p.count + mt) : "memory");
                }
            }
            // wait for every tile of the row block, then the row's scale
            bool done = true;
            if (et == 0) done = wait_count(p.count + mt, (uint32_t)p.n_t, abort_flag, p.status, SITE_E_ROWS);
            if (!named_bar_and(1, kEpiThreads, done)) break;
            const float amax = row_ok ? __uint_as_float(ld_acquire_gpu(p.amax + gm)) : 0.0f;
            float scale, inv;
            absmax_scales(amax, scale, inv);
            if (nt == 0 && slice == 0 && row_ok) p.s_tok_out[gm] = scale;
            // pass 2: codes from the registers, one 32x32 box per chunk through
            // shared memory to a TMA store (rows >= M and columns >= N clipped)
            const uint64_t inv2 = f2_splat(inv);
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                uint32_t w[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) w[q] = quant4_packed(h[c][2 * q], h[c][2 * q + 1], inv2);
                if (lane == 0) bulk_wait_read_all();   // the box's previous store has read it
                __syncwarp();
                stage_row_swizzled<32>(stg, lane, w);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, stg_s, nt * BN + slice * 64 + c * CW, mt * BM + quarter * 32);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all();   // this warp's TMA stores have landed
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// Zeroes the absmax words and row-block counters of the requantizing linear.
// It lets the linear launch at once (its prologue and first weight loads then
// overlap this kernel and the one before it) but waits for the previous grid
// before writing (an earlier call may still read the words).
__global__ void zero_words_kernel(uint32_t* __restrict__ w, int n) {
    griddep_launch_dependents();
    griddep_wait();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) w[i] = 0u;
}

constexpr int kMaxDevices = 64;

}  // namespace

size_t requant_grid_scratch_bytes(int64_t T) {
    const int64_t m_tiles = (T + BM - 1) / BM;
    return (size_t)(T + m_tiles) * sizeof(uint32_t);
}

int launch_w8a8_requant_grid(const LinearArgs& a, uint32_t* scratch, size_t scratch_bytes, const DeviceInfo& di,
                             cudaStream_t st) {
    static_assert(smem_bytes() <= 232448, "shared memory budget");
    static_assert(smem_bytes() > 116 * 1024, "one CTA per SM (it owns all of TMEM)");
    const int64_t n_t = (a.N + BN - 1) / BN;
    const int64_t m_tiles = (a.T + BM - 1) / BM;
    const int64_t tiles = n_t * m_tiles;
    const int grid = (int)(tiles < di.sm_count ? tiles : di.sm_count);
    // every wait ends only if a row block's tiles fit in one pass over the grid
    if (a.T <= 64 || n_t > grid) return ZQ_ERR_SHAPE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    auto kern = w8a8_requant_grid_kernel;
    const size_t smem = smem_bytes();
    int rc;
    {
        static bool attr_set[kMaxDevices] = {};
        static int per_sm[kMaxDevices] = {};
        std::lock_guard<std::mutex> lk(launch_cache_mutex());
        if (!attr_set[dev]) {
            if ((rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))))
                return rc;
            if ((rc = cuda_status(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm[dev], kern, kThreads, smem))))
                return rc;
            attr_set[dev] = true;
        }
        // the CTAs wait on one another: all of them must be resident at once
        if (per_sm[dev] < 1) return ZQ_ERR_SHAPE;
    }
    if (!scratch || scratch_bytes < requant_grid_scratch_bytes(a.T)) return ZQ_ERR_WORKSPACE;
    uint32_t* amax = scratch;
    uint32_t* count = scratch + a.T;
    const int nwords = (int)(a.T + m_tiles);
    {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        cfg.attrs = at;
        cfg.numAttrs = (unsigned)pdl_attr(at[0]);
        const int blocks = (nwords + 255) / 256;
        cfg.gridDim = dim3((unsigned)(blocks < di.sm_count ? blocks : di.sm_count));
        cfg.blockDim = dim3(256);
        cfg.stream = st;
        count_launch();
        if ((rc = cuda_status(cudaLaunchKernelEx(&cfg, zero_words_kernel, scratch, nwords)))) return rc;
    }
    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_i8(&ta, a.xq, a.T, a.K, BM))) return rc;
    if ((rc = make_tmap_i8(&tb, a.Wq, a.N, a.K, BN))) return rc;
    if ((rc = make_tmap_out(&ty, a.y, a.T, a.N, 1))) return rc;
    Params p{};
    p.M = (int)a.T;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.G = (int)a.G;
    p.n_t = (int)n_t;
    p.m_tiles = (int)m_tiles;
    p.s_tok = a.s_tok;
    p.s_grp = a.s_grp;
    p.bias = a.bias;
    p.s_tok_out = a.s_tok_out;
    p.amax = amax;
    p.count = count;
    p.act = a.act;
    p.status = di.status_word;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
}

}  // namespace zq
