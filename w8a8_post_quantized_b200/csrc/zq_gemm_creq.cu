// zq_gemm_creq.cu -- W8A8 linear whose epilogue requantizes the output per
// token for the next layer, with no scratch memory: dequantize + bias + GeLU,
// per-token absmax over the whole output row, per-token scale, int8 codes.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (the fused "GEMM + DeQuantize"
// kernel feeding the next op; token-wise quantization fused with the op that
// produces the activations) and "探秘Transformer系列之（36）— 大模型量化方案"
// §1.2.2 (INT32 accumulators scaled by the weight and activation scales before
// the next op; one dynamic scale per token).
//
// The per-token scale needs the absmax of a whole output row, which spans
// N / 256 accumulator tiles.  Here a thread-block cluster of C CTAs owns a
// block of 128 rows and all N columns: CTA `rank` computes column tiles
// 2*rank and 2*rank+1 into its two TMEM accumulators (512 columns, the whole
// TMEM).  The epilogue
//   pass 1  dequantizes, adds bias, applies GeLU (packed fp32 pair arithmetic),
//           writes the fp32 result back into TMEM in place (tcgen05.st) and
//           keeps a per-row partial absmax;
//   xchg    pushes each row's partial absmax into every cluster CTA's shared
//           memory with asynchronous distributed-shared-memory stores that
//           count their bytes on the receiver's exchange mbarrier; waits until
//           all C partials of its own rows have landed;
//   pass 2  reads the fp32 result back from TMEM and writes int8 codes with
//           scale = absmax/127, code = rint(fl(h * fl(127/absmax))).
// The producer (TMA) and MMA warps are those of the plain kernel; the tile
// order walks the cluster's row blocks.  Every wait is bounded.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int UMMA_K = 32;
constexpr int EW = 16;                         // epilogue warps
constexpr int kThreads = 64 + 32 * EW;
constexpr int kEpiThreads = 32 * EW;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr int kMaxCluster = 8;
constexpr uint32_t kTmemCols = 512;

enum {
    SITE_P_EMPTY = 0x501,
    SITE_P_DRAIN = 0x502,
    SITE_M_TEMPTY = 0x503,
    SITE_M_FULL = 0x504,
    SITE_M_DRAIN = 0x505,
    SITE_E_TFULL = 0x506,
    SITE_E_XCHG = 0x507,
};

struct Params {
    int M, N, K, G;
    int C;                 // CTAs per cluster (= ceil(n_tiles / 2))
    const float* s_tok;
    const float* s_grp;
    const float* bias;     // may be null
    int8_t* y;             // [M, N]
    float* s_tok_out;      // [M]
    int act;
    int* status;
};

template <int STAGES, int NSTG>
__host__ __device__ constexpr size_t smem_bytes() {
    // ring + int8 output staging (NSTG 32x32 boxes per epilogue warp) + barriers/
    // flags (256) + column factors [2 halves][scale, bias][BN] + per-slice row
    // partials [4][BM] + exchange [2][kMaxCluster][BM]
    return 1024 + (size_t)STAGES * (A_STAGE + B_STAGE) + NSTG * EW * 32 * 32 + 256 + 2 * 2 * BN * 4 + 4 * BM * 4 +
           2 * kMaxCluster * BM * 4;
}

// Pass 1 on one 32-column chunk of one row, in place: accumulators (int32
// words) in, y = s_tok * s_grp * acc + bias (+GeLU) as fp32 words out, in
// packed pair arithmetic.  UNI: the chunk lies in one weight group, so the
// combined scale is one number.
template <bool GELU, bool UNI>
__device__ __forceinline__ void pass1_chunk(uint32_t (&v)[32], float row_scale, const float* scc,
                                            const float* bic, float& pmax) {
    uint64_t f[16];
    dequant_chunk<GELU, UNI>(v, row_scale, scc, bic, nullptr, 0, f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float t0, t1;
        f2_unpack(f[i], t0, t1);
        pmax = fmaxf(pmax, fmaxf(fabsf(t0), fabsf(t1)));
        v[2 * i] = __float_as_uint(t0);
        v[2 * i + 1] = __float_as_uint(t1);
    }
}

template <int STAGES, int NSTG>
__global__ void __launch_bounds__(kThreads, 1)
w8a8_requant_cluster_kernel(const __grid_constant__ CUtensorMap tmA,
                            const __grid_constant__ CUtensorMap tmB,
                            const __grid_constant__ CUtensorMap tmY, const Params p) {
    constexpr uint32_t IDESC = idesc_i8(BM, BN);
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * A_STAGE;
    const uint32_t sStg = sB + STAGES * B_STAGE;  // [EW][NSTG][32 rows][32 B], 1024-aligned
    const uint32_t sBar = sStg + NSTG * EW * 32 * 32;
    uint8_t* gBar = gbase + (sBar - base);
    // barriers: full[S], empty[S], tfull[2], tempty[2], drain, xbar[2]
    auto bar_full = [&](int s) { return sBar + 8u * s; };
    auto bar_empty = [&](int s) { return sBar + 8u * (STAGES + s); };
    auto bar_tfull = [&](int b) { return sBar + 8u * (2 * STAGES + b); };
    auto bar_tempty = [&](int b) { return sBar + 8u * (2 * STAGES + 2 + b); };
    const uint32_t bar_drain = sBar + 8u * (2 * STAGES + 4);
    auto bar_xchg = [&](int b) { return sBar + 8u * (2 * STAGES + 5 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 7));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* col_f = reinterpret_cast<float*>(gBar + 256);                 // [2][2][BN]
    float* slice_part = col_f + 2 * 2 * BN;                              // [4][BM]
    uint32_t* xch = reinterpret_cast<uint32_t*>(slice_part + 4 * BM);    // [2][kMaxCluster][BM]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int rank = (int)cluster_ctarank();
    const int cl = (int)cluster_id_x();
    const int ncl = (int)cluster_count_x();
    const int m_tiles = (p.M + BM - 1) / BM;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int kblocks = (p.K + BK - 1) / BK;
    const bool real0 = 2 * rank < n_tiles;       // does this CTA own column tile 2*rank (half 0)?
    const bool real1 = 2 * rank + 1 < n_tiles;   // ... and 2*rank+1 (half 1)?

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull(b), 1);
            mbar_init(bar_tempty(b), EW);
            mbar_init(bar_xchg(b), 1);     // the local expect-tx arrival; peers' bytes complete it
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
    cluster_sync_all();  // every CTA's exchange barriers are initialised before any peer arrives
    griddep_wait();      // inputs and outputs are free of the previous grid in the stream
    griddep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int mb = cl; ok && mb < m_tiles; mb += ncl) {
                for (int h = 0; ok && h < 2; ++h) {
                    if (!(h ? real1 : real0)) continue;
                    const int nt = 2 * rank + h;
                    for (int kb = 0; kb < kblocks; ++kb, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait(bar_empty(s), ph ^ 1u, abort_flag, p.status, SITE_P_EMPTY)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_full(s), A_STAGE + B_STAGE);
                        tma_load_2d(sA + s * A_STAGE, &tmA, bar_full(s), kb * BK, mb * BM);
                        tma_load_2d(sB + s * B_STAGE, &tmB, bar_full(s), kb * BK, nt * BN);
                    }
                }
            }
            const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(bar_full(j % STAGES), (j / STAGES) & 1u, nullptr, p.status, SITE_P_DRAIN);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, mbi = 0;
            bool ok = true;
            for (int mb = cl; ok && mb < m_tiles; mb += ncl, ++mbi) {
                for (int h = 0; ok && h < 2; ++h) {
                    if (!(h ? real1 : real0)) continue;
                    // accumulator h is used once per row block: phase = mbi & 1
                    if (!mbar_wait(bar_tempty(h), (mbi & 1u) ^ 1u, abort_flag, p.status, SITE_M_TEMPTY)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t d_tmem = tmem_base + (uint32_t)(h * BN);
                    for (int kb = 0; kb < kblocks; ++kb, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
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
                    if (ok) mma_commit(bar_tfull(h));
                }
            }
            mma_commit(bar_drain);
            mbar_wait(bar_drain, 0u, nullptr, p.status, SITE_M_DRAIN);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        constexpr int SLICES = EW / 4;
        constexpr int CW = 32;
        constexpr int CT = BN / CW;
        const int quarter = warp & 3;
        const int slice = (warp - 2) >> 2;
        const int c_begin = slice * CT / SLICES, c_end = (slice + 1) * CT / SLICES;
        const int r = quarter * 32 + lane;
        const int et = threadIdx.x - 64;
        uint8_t* stg0 = gbase + (sStg - base) + (uint32_t)(warp - 2) * NSTG * 32u * 32u;  // this warp's boxes
        const bool gelu = p.act == ZQ_ACT_GELU;
        const bool uni = p.G % CW == 0;  // every 32-column chunk lies in one weight group
        // This CTA's columns are the same for every row block: stage their
        // weight-group scales and biases once.
        for (int i = et; i < 2 * BN; i += kEpiThreads) {
            const int h = i / BN, c = i % BN;
            const int n = (2 * rank + h) * BN + c;
            const bool in = n < p.N;
            col_f[h * 2 * BN + c] = in ? __ldg(p.s_grp + n / p.G) : 0.0f;
            col_f[h * 2 * BN + BN + c] = (in && p.bias) ? __ldg(p.bias + n) : 0.0f;
        }
        named_bar_sync(1, kEpiThreads);
        float next_scale = (cl < m_tiles && cl * BM + r < p.M) ? __ldg(p.s_tok + cl * BM + r) : 0.0f;
        uint32_t mbi = 0;
        for (int mb = cl; mb < m_tiles; mb += ncl, ++mbi) {
            const int gm = mb * BM + r;
            const bool row_ok = gm < p.M;
            const float row_scale = next_scale;  // loaded one row block ahead
            const int gn = gm + ncl * BM;
            next_scale = (mb + ncl < m_tiles && gn < p.M) ? __ldg(p.s_tok + gn) : 0.0f;

            // pass 1: y = dequant + bias (+GeLU); written back to TMEM; partial
            // absmax.  Warps go at their own pace; a failed wait is carried to the
            // exchange barrier below, where all epilogue threads agree on it.
            float pmax = 0.0f;
            bool ok = true;
            for (int h = 0; ok && h < 2; ++h) {
                if (!(h ? real1 : real0)) continue;
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(bar_tfull(h), mbi & 1u, abort_flag, p.status, SITE_E_TFULL));
                if (!ok) break;
                tc_fence_after();
                const float* sc = col_f + h * 2 * BN;
                const float* bi = sc + BN;
                const uint32_t t_row = tmem_base + (uint32_t)(h * BN) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
                for (int c = c_begin; c < c_end; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + c * CW, v);
                    tmem_ld_wait();
                    const float* scc = sc + c * CW;
                    const float* bic = bi + c * CW;
                    if (gelu) {
                        if (uni) pass1_chunk<true, true>(v, row_scale, scc, bic, pmax);
                        else pass1_chunk<true, false>(v, row_scale, scc, bic, pmax);
                    } else {
                        if (uni) pass1_chunk<false, true>(v, row_scale, scc, bic, pmax);
                        else pass1_chunk<false, false>(v, row_scale, scc, bic, pmax);
                    }
                    tmem_st_32x32b_x32(t_row + c * CW, v);
                }
                tmem_st_wait();
            }

            // exchange: row absmax over this CTA's column slices, then over the cluster
            // Each CTA's exchange barrier expects C * BM * 4 bytes per use; every
            // cluster CTA sends its BM row partials with asynchronous stores that
            // count on the receiver's barrier.  Buffer `buf` is rewritten two row
            // blocks later, by which time every receiver has read it: a sender
            // gets there only after its own barrier for the next block completed,
            // which needs every CTA's next-block partials, sent after reading.
            const int buf = mbi & 1;
            slice_part[slice * BM + r] = pmax;
            if (et == 0 && ok) mbar_arrive_expect_tx(bar_xchg(buf), (uint32_t)(p.C * BM * 4));
            if (!named_bar_and(1, kEpiThreads, ok)) break;
            if (slice == 0) {
                float m = slice_part[r];
#pragma unroll
                for (int s = 1; s < SLICES; ++s) m = fmaxf(m, slice_part[s * BM + r]);
                const uint32_t local = smem_u32(xch + (buf * kMaxCluster + rank) * BM + r);
                for (int q = 0; q < p.C; ++q)
                    st_async_u32(mapa_shared(local, (uint32_t)q), __float_as_uint(m),
                                 mapa_shared(bar_xchg(buf), (uint32_t)q));
            }
            const bool got = mbar_wait_cluster(bar_xchg(buf), (mbi >> 1) & 1u, abort_flag, p.status, SITE_E_XCHG);
            if (!named_bar_and(1, kEpiThreads, got)) break;
            float amax = 0.0f;
            for (int q = 0; q < p.C; ++q) amax = fmaxf(amax, __uint_as_float(xch[(buf * kMaxCluster + q) * BM + r]));
            float scale, inv;
            absmax_scales(amax, scale, inv);
            if (rank == 0 && slice == 0 && row_ok) p.s_tok_out[gm] = scale;

            // pass 2: codes from the fp32 values kept in TMEM
            const uint64_t inv2 = f2_splat(inv);  // codes: fl(fl(h * inv) + 1.5*2^23), two roundings
            int kst = 0;                       // staging box in turn
            for (int h = 0; h < 2; ++h) {
                if (!(h ? real1 : real0)) continue;
                const uint32_t t_row = tmem_base + (uint32_t)(h * BN) + ((uint32_t)(quarter * 32) << 16);
#pragma unroll 1
                for (int c = c_begin; c < c_end; ++c) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + c * CW, v);
                    tmem_ld_wait();
                    const int n0 = (2 * rank + h) * BN + c * CW;
                    uint32_t w[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q)
                        w[q] = quant4_packed(u2_pack(v[4 * q], v[4 * q + 1]), u2_pack(v[4 * q + 2], v[4 * q + 3]), inv2);
                    // the warp's 32x32 box of codes: shared memory, then one TMA store
                    // (rows >= M and columns >= N are clipped); the box's previous
                    // store (NSTG boxes ago) must have finished reading it
                    uint8_t* stg = stg0 + kst * 32 * 32;
                    const uint32_t stg_s = smem_u32(stg);
                    kst = kst + 1 == NSTG ? 0 : kst + 1;
                    if (lane == 0) {
                        if (NSTG == 2) bulk_wait_read_1();
                        else bulk_wait_read_all();
                    }
                    __syncwarp();
                    stage_row_swizzled<32>(stg, lane, w);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmY, stg_s, n0, mb * BM + quarter * 32);
                        bulk_commit();
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_tempty(h));
            }
        }
        if (lane == 0) bulk_wait_all();  // this warp's TMA stores have landed
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync_all();  // no CTA leaves while a peer may still write its shared memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

constexpr int kStages = 4;
constexpr int kStg = 1;
constexpr int kMaxDevices = 64;

}  // namespace

int launch_w8a8_requant_cluster(const LinearArgs& a, const DeviceInfo& di, cudaStream_t st) {
    static_assert(smem_bytes<kStages, kStg>() <= 232448, "shared memory budget");
    static_assert(smem_bytes<kStages, kStg>() > 116 * 1024, "one CTA per SM (TMEM ownership)");
    const int64_t n_tiles = (a.N + BN - 1) / BN;
    const int C = (int)((n_tiles + 1) / 2);
    if (a.T <= 64 || C < 1 || C > kMaxCluster) return ZQ_ERR_SHAPE;
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    auto kern = w8a8_requant_cluster_kernel<kStages, kStg>;
    const size_t smem = smem_bytes<kStages, kStg>();
    static bool attr_set[kMaxDevices] = {};
    static int max_clusters[kMaxDevices][kMaxCluster + 1] = {};
    int rc;
    std::unique_lock<std::mutex> lk(launch_cache_mutex());
    if (!attr_set[dev]) {
        if ((rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem))))
            return rc;
        attr_set[dev] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    if (max_clusters[dev][C] == 0) {
        cfg.gridDim = dim3(C);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();  // clear; the caller falls back to the scratch path
            max_clusters[dev][C] = -1;
        } else {
            max_clusters[dev][C] = n;
        }
    }
    const int max_ncl = max_clusters[dev][C];
    lk.unlock();
    if (max_ncl < 1) return ZQ_ERR_SHAPE;
    const int64_t m_tiles = (a.T + BM - 1) / BM;
    const int ncl = (int)(m_tiles < max_ncl ? m_tiles : max_ncl);
    cfg.gridDim = dim3(ncl * C);
    cfg.numAttrs = 1 + (unsigned)pdl_attr(attr[1]);

    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_i8(&ta, a.xq, a.T, a.K, BM))) return rc;
    if ((rc = make_tmap_i8(&tb, a.Wq, a.N, a.K, BN))) return rc;
    if ((rc = make_tmap_out(&ty, a.y, a.T, a.N, 1))) return rc;
    Params p{};
    p.M = (int)a.T;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.G = (int)a.G;
    p.C = C;
    p.s_tok = a.s_tok;
    p.s_grp = a.s_grp;
    p.bias = a.bias;
    p.y = static_cast<int8_t*>(a.y);
    p.s_tok_out = a.s_tok_out;
    p.act = a.act;
    p.status = di.status_word;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
}

}  // namespace zq
