// zq_gemm.cu -- W8A8 linear for sm_100a: INT8 x INT8 -> INT32 on the
// 5th-generation tensor cores (tcgen05.mma kind::i8) with the
// dequantization epilogue fused.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (the fused "GEMM + DeQuantize"
// kernel) and "探秘Transformer系列之（36）— 大模型量化方案" §1.2.2 (the INT32
// accumulation is scaled by the activation and weight scales before the
// result is written for the next op) and §1.1.2 (denormalisation by the outer
// product of the per-row and per-column scales).  The pages' kernel targets
// Ampere (WMMA tiles via CUTLASS, group size tuned to 16/32); here groups are
// whole output rows, so the scale of an output column is constant along K and
// the whole contraction stays in exact int32 on the tensor core, with the
// scales applied once per output element in the epilogue.
//
// Structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: 128-row x 128-byte tiles of both operands into
//               a STAGES-deep shared-memory ring (128-byte swizzle), one
//               mbarrier per stage counting the bytes that landed;
//   warp 1      allocates TMEM, then one thread issues tcgen05.mma (M=128,
//               N=BN, K=32 per instruction, 4 per stage) into one of two
//               TMEM accumulators and commits stage release / tile-done
//               mbarriers;
//   warps 2..5  epilogue: tcgen05.ld of the int32 accumulator (each warp
//               owns its 32-lane quarter of TMEM), dequantize with the
//               token and group scales, add bias, optional GeLU, store
//               fp32 / bf16 / int32, or fp32 plus a per-row absmax for
//               requantization.  Two accumulators let the epilogue of tile
//               i overlap the main loop of tile i+1.
// Operand roles: normally the M side is the activations (rows = tokens) and
// the N side the weights; for few tokens (decode) the roles swap so the
// weights fill the 128-row MMA side and the tokens become N = 16..64.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int BM = 128;         // MMA M: rows of the M-side operand per tile
constexpr int BK = 128;         // K bytes per pipeline stage (one swizzle row)
constexpr int UMMA_K = 32;      // K per tcgen05.mma of kind::i8
// block = 2 warps (TMA producer, MMA issuer) + EW epilogue warps
template <int EW>
__host__ __device__ constexpr int block_threads() { return 64 + 32 * EW; }
constexpr int A_STAGE = BM * BK;

enum Epi { EPI_I32 = 0, EPI_F32 = 1, EPI_BF16 = 2, EPI_REQ = 3 };

// Status sites recorded when a bounded wait expires.
enum WaitSite {
    SITE_PRODUCER_EMPTY = 0x101,
    SITE_MMA_TMEM_EMPTY = 0x201,
    SITE_MMA_FULL = 0x202,
    SITE_MMA_DRAIN = 0x203,
    SITE_EPI_TMEM_FULL = 0x301,
    SITE_PRODUCER_DRAIN = 0x102,
};

struct Params {
    int M, N, K;        // kernel roles: M-side rows, N-side rows, reduction length
    int G;              // weight rows per scale group
    int ldy;            // row length of y (= number of output features)
    const float* s_tok;
    const float* s_grp;
    const float* bias;  // may be null
    void* y;
    uint32_t* amax;     // EPI_REQ: per-token absmax bits
    int act;
    int group_m;        // tile raster: groups of group_m row tiles sweep all column tiles
    int* status;
    // LLM.int8() outlier part (OUTL kernels): fp16 [M, 8] activations and
    // fp16 [N, 8] weights of the decomposed columns (zeros past the count)
    const uint16_t* xo;
    const uint16_t* wo;
};

// Tile index -> (row tile, column tile).  Tiles run in groups of GM row tiles:
// inside a group the row tile varies fastest, then the column tile, so the
// group's slice of the M-side operand stays in L2 while every column tile
// of the other operand streams past it once per group.
__device__ __forceinline__ void tile_coords(int tile, int m_tiles, int n_tiles, int GM, int& mt, int& nt) {
    const int per_group = GM * n_tiles;
    const int g = tile / per_group;
    const int rem = tile - g * per_group;
    const int gm = min(GM, m_tiles - g * GM);  // the last group may be short
    mt = g * GM + rem % gm;
    nt = rem / gm;
}

template <int BN>
__host__ __device__ constexpr uint32_t tmem_cols() {
    return (2 * BN <= 32) ? 32 : (2 * BN <= 64) ? 64 : (2 * BN <= 128) ? 128 : (2 * BN <= 256) ? 256 : 512;
}

// Bytes of one 32x32 output box row: int32/fp32 outputs 128, bf16 64.
template <int EPI>
__host__ __device__ constexpr int out_row_bytes() { return EPI == EPI_BF16 ? 64 : 128; }

template <int BN, int STAGES, bool SWAP, int EPI, int EW>
__host__ __device__ constexpr size_t smem_bytes() {
    // 1024 alignment slack + operand ring + output staging (one 32x32 box per
    // epilogue warp, non-swapped only) + barriers/flags + per-column factors
    // (bf16 outputs stage only the per-column scale; their bias is read
    // through L1, which leaves room for a fourth pipeline stage at BN = 256)
    // (swapped kernels: two int32 partial-accumulator buffers for split-K)
    return 1024 + (size_t)STAGES * (A_STAGE + BN * BK) +
           (SWAP ? (size_t)2 * BM * BN * 4 : (size_t)EW * 32 * out_row_bytes<EPI>()) + 256 +
           (EPI == EPI_I32 ? 0 : EPI == EPI_BF16 && !SWAP ? 1 : 2) * BN * sizeof(float);
}

template <int BN, int STAGES, bool SWAP, int EPI, int EW, bool OUTL = false>
__global__ void __launch_bounds__(block_threads<EW>(), 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const Params p) {
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M=128 is 16..256 step 16");
    static_assert(EW % 4 == 0 && EW >= 4 && EW <= 16, "epilogue warps cover the 4 TMEM lane quarters");
    static_assert(!OUTL || (!SWAP && (EPI == EPI_F32 || EPI == EPI_BF16)), "outlier part: fp32/bf16 tiles");
    constexpr int kEpiThreads = 32 * EW;
    constexpr int B_STAGE = BN * BK;
    // epilogue column chunk (16 for the swapped 32-token tile: 32 there spills
    // registers next to the split-K partial sums)
    constexpr int CW = (BN % 32 == 0 && !(SWAP && BN == 32)) ? 32 : 16;
    constexpr uint32_t IDESC = idesc_i8(BM, BN);
    constexpr uint32_t TMEM_COLS = tmem_cols<BN>();

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    constexpr int RB = out_row_bytes<EPI>();
    constexpr uint32_t STG_BYTES = SWAP ? 0u : (uint32_t)EW * 32u * RB;
    const uint32_t sA = base;
    const uint32_t sB = base + STAGES * A_STAGE;
    const uint32_t sStg = sB + STAGES * B_STAGE;  // 1024-aligned: every stage is a multiple of 1024
    // swapped: split-K partials [2 buffers][BM rows][BN] int32 (in place of the staging boxes)
    const uint32_t sPart = sStg;
    const uint32_t sBar = sStg + (SWAP ? 2u * BM * BN * 4u : STG_BYTES);
    uint8_t* gBar = gbase + (sBar - base);
    // barrier layout: full[S], empty[S], tfull[2], tempty[2], drain
    auto bar_full = [&](int s) { return sBar + 8u * s; };
    auto bar_empty = [&](int s) { return sBar + 8u * (STAGES + s); };
    auto bar_tfull = [&](int b) { return sBar + 8u * (2 * STAGES + b); };
    auto bar_tempty = [&](int b) { return sBar + 8u * (2 * STAGES + 2 + b); };
    const uint32_t bar_drain = sBar + 8u * (2 * STAGES + 4);
    // split-K (swapped): partials of buffer b are ready at the leader / free again at a peer
    auto bar_red_full = [&](int b) { return sBar + 8u * (2 * STAGES + 5 + b); };
    auto bar_red_free = [&](int b) { return sBar + 8u * (2 * STAGES + 7 + b); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 9));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    float* stage_f = reinterpret_cast<float*>(gBar + 256);  // [2][BN]

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // swapped kernels run as clusters of S CTAs splitting K (S may be 1);
    // the others as independent CTAs
    const int S = SWAP ? (int)cluster_size() : 1;
    const int rank = SWAP ? (int)cluster_ctarank() : 0;
    const int cl = SWAP ? (int)cluster_id_x() : (int)blockIdx.x;
    const int ncl = SWAP ? (int)cluster_count_x() : (int)gridDim.x;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_tfull(b), 1);
            mbar_init(bar_tempty(b), EW);
            if (SWAP) {
                mbar_init(bar_red_full(b), S > 1 ? S - 1 : 1);
                mbar_init(bar_red_free(b), 1);
            }
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_proxy_async_smem();
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (!SWAP) tma_prefetch_desc(&tmY);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (SWAP) cluster_sync_all();  // peers' barriers initialised before any remote arrive
    // Programmatic dependent launch.  The weights (codes, group scales, bias)
    // are never written by a kernel that lets its successor start early (the
    // hot-path kernels that trigger early write only activations and outputs;
    // the weight preparation kernels run to completion first), so the
    // producer streams the first ring of weight tiles before waiting for the
    // previous grid; every role waits before it touches activations or
    // outputs.
    griddep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;

    const int m_tiles = (p.M + BM - 1) / BM;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = m_tiles * n_tiles;
    const int kblocks_all = (p.K + BK - 1) / BK;
    // this CTA's share of the K loop (the whole loop unless split)
    const int kb_begin = rank * kblocks_all / S;
    const int kb_end = (rank + 1) * kblocks_all / S;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            // the weight operand is A when the roles are swapped, else B
            auto load_w = [&](int s, int kb, int mt, int nt) {
                if (SWAP) tma_load_2d(sA + s * A_STAGE, &tmA, bar_full(s), kb * BK, mt * BM);
                else tma_load_2d(sB + s * B_STAGE, &tmB, bar_full(s), kb * BK, nt * BN);
            };
            auto load_x = [&](int s, int kb, int mt, int nt) {
                if (SWAP) tma_load_2d(sB + s * B_STAGE, &tmB, bar_full(s), kb * BK, nt * BN);
                else tma_load_2d(sA + s * A_STAGE, &tmA, bar_full(s), kb * BK, mt * BM);
            };
            // first ring fill: the weight halves of the first STAGES stages
            // (their slots are free), before the wait for the previous grid
            uint32_t npre = 0;
            for (int tile = cl; npre < (uint32_t)STAGES && tile < num_tiles; tile += ncl) {
                int mt, nt;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt, nt);
                for (int kb = kb_begin; kb < kb_end && npre < (uint32_t)STAGES; ++kb, ++npre) {
                    mbar_arrive_expect_tx(bar_full((int)npre), A_STAGE + B_STAGE);
                    load_w((int)npre, kb, mt, nt);
                }
            }
            griddep_wait();
            uint32_t it = 0;
            bool ok = true;
            for (int tile = cl; ok && tile < num_tiles; tile += ncl) {
                int mt, nt;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt, nt);
                for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (it >= npre) {
                        if (!mbar_wait(bar_empty(s), ph ^ 1u, abort_flag, p.status, SITE_PRODUCER_EMPTY)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_full(s), A_STAGE + B_STAGE);
                        load_w(s, kb, mt, nt);
                    }
                    load_x(s, kb, mt, nt);
                }
            }
            // Let every copy this thread issued land before the CTA can exit:
            // wait on the most recent phase of each stage that was used.
            const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
            for (uint32_t j = first; j < it; ++j)
                mbar_wait(bar_full(j % STAGES), (j / STAGES) & 1u, nullptr, p.status,
                          SITE_PRODUCER_DRAIN);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t it = 0, lt = 0;
            bool ok = true;
            for (int tile = cl; ok && tile < num_tiles; tile += ncl, ++lt) {
                const int b = lt & 1;
                const uint32_t tph = (lt >> 1) & 1u;
                if (!mbar_wait(bar_tempty(b), tph ^ 1u, abort_flag, p.status, SITE_MMA_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * BN);
                for (int kb = kb_begin; kb < kb_end; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1u;
                    if (!mbar_wait(bar_full(s), ph, abort_flag, p.status, SITE_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sdesc_k_sw128(sA + s * A_STAGE);
                    const uint64_t db = sdesc_k_sw128(sB + s * B_STAGE);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k)
                        // +32 bytes along K inside the swizzle atom = +2 in the
                        // descriptor's (address >> 4) field
                        mma_i8(d_tmem, da + 2u * k, db + 2u * k, IDESC, (kb > kb_begin || k > 0) ? 1u : 0u);
                    mma_commit(bar_empty(s));  // stage free once these MMAs finish
                }
                if (ok) mma_commit(bar_tfull(b));  // accumulator b complete
            }
            // All MMAs issued by this thread complete before teardown.
            mma_commit(bar_drain);
            mbar_wait(bar_drain, 0u, nullptr, p.status, SITE_MMA_DRAIN);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------ epilogue
        griddep_wait();  // token scales are the previous grid's output; y may still be read by it
        // warp w may only read TMEM lanes 32*(w%4) .. +31; EW/4 warps share each
        // lane quarter and split the tile's columns between them
        constexpr int SLICES = EW / 4;
        constexpr int CT = BN / CW;             // column chunks per tile
        const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
        const int slice = (warp - 2) >> 2;      // which share of the columns
        const int c_begin = slice * CT / SLICES, c_end = (slice + 1) * CT / SLICES;
        const int r = quarter * 32 + lane;      // row of the tile this thread owns
        const int et = threadIdx.x - 64;        // 0 .. 32*EW-1
        uint8_t* stg = gbase + (sStg - base) + (uint32_t)(warp - 2) * 32u * RB;  // this warp's box
        const uint32_t stg_s = smem_u32(stg);
        (void)stg;
        (void)stg_s;
        const bool gelu = p.act == ZQ_ACT_GELU;
        if constexpr (!SWAP) {
            // Each warp runs on its own (no CTA-wide barrier per tile): it waits
            // for the accumulator, converts its chunks and frees the accumulator
            // with its own arrival.  The column factors of the next chunk it will
            // handle (lane l: scale and bias of column l) and the token scale of
            // its next tile are loaded one step ahead, so their latency hides
            // behind the current chunk.
            const bool uni = p.G % 32 == 0;  // each 32-column chunk lies in one weight group
            float pa = 0.0f, pb = 0.0f, prs = 0.0f;
            auto fetch_cols = [&](int tile, int c) {
                int mt_, nt_;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt_, nt_);
                const int n = nt_ * BN + c * CW + lane;
                const bool in = n < p.N;
                pa = in ? __ldg(p.s_grp + n / p.G) : 0.0f;
                pb = (in && p.bias) ? __ldg(p.bias + n) : 0.0f;
            };
            auto fetch_row = [&](int tile) {
                int mt_, nt_;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt_, nt_);
                const int gm = mt_ * BM + r;
                prs = gm < p.M ? __ldg(p.s_tok + gm) : 0.0f;
            };
            if (EPI != EPI_I32 && cl < num_tiles) {
                fetch_cols(cl, c_begin);
                fetch_row(cl);
            }
            uint32_t lt = 0;
            for (int tile = cl; tile < num_tiles; tile += ncl, ++lt) {
                int mt, nt;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt, nt);
                const int b = lt & 1;
                const uint32_t tph = (lt >> 1) & 1u;
                const float row_scale = prs;
                if (EPI != EPI_I32 && tile + ncl < num_tiles) fetch_row(tile + ncl);
                // the warp's lanes take one decision, so none waits alone later
                const bool got = mbar_wait(bar_tfull(b), tph, abort_flag, p.status, SITE_EPI_TMEM_FULL);
                if (!__all_sync(0xFFFFFFFFu, got)) break;
                tc_fence_after();
                const int gm = mt * BM + r;  // token row owned by this thread
                const bool row_ok = gm < p.M;
                float amax = 0.0f;
                float xo[8];  // this token's outlier activations (OUTL)
                if constexpr (OUTL) {
                    uint4 u = make_uint4(0u, 0u, 0u, 0u);
                    if (row_ok) u = __ldg(reinterpret_cast<const uint4*>(p.xo) + gm);
                    const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        xo[2 * q] = half_lo(uw[q]);
                        xo[2 * q + 1] = half_hi(uw[q]);
                    }
                }
                const uint32_t t_row = tmem_base + (uint32_t)(b * BN) + ((uint32_t)(quarter * 32) << 16);
                static_assert(SWAP || CW == 32, "non-swapped tiles are whole 32-column chunks");
#pragma unroll 1
                for (int c = c_begin; c < c_end; ++c) {
                    const float ca = pa, cb = pb;
                    if (EPI != EPI_I32) {
                        if (c + 1 < c_end) fetch_cols(tile, c + 1);
                        else if (tile + ncl < num_tiles) fetch_cols(tile + ncl, c_begin);
                    }
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(t_row + c * CW, v);
                    tmem_ld_wait();
                    const int n0 = nt * BN + c * CW;  // first column of the chunk
                    // thread owns token gm (box row `lane`), columns n0 .. n0+31; the
                    // warp's 32x32 box goes through shared memory to one TMA store
                    // (rows >= M and columns >= N are clipped by the store)
                    uint32_t w[RB / 4];
                    if constexpr (EPI == EPI_I32) {
#pragma unroll
                        for (int j = 0; j < 32; ++j) w[j] = v[j];
                    } else {
                        uint64_t f[16];
                        if constexpr (OUTL) {
                            // the chunk's outlier weight columns, transposed ([k][column])
                            // into this warp's staging box once its previous store has read it
                            uint4 u = make_uint4(0u, 0u, 0u, 0u);
                            if (n0 + lane < p.N) u = __ldg(reinterpret_cast<const uint4*>(p.wo) + n0 + lane);
                            if (lane == 0) bulk_wait_read_all();
                            __syncwarp();
                            float* box = reinterpret_cast<float*>(stg);
                            const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                box[(2 * q) * 32 + lane] = half_lo(uw[q]);
                                box[(2 * q + 1) * 32 + lane] = half_hi(uw[q]);
                            }
                            __syncwarp();
                            if (gelu) {
                                if (uni) dequant_chunk_lanes_outl<true, true>(v, row_scale, ca, cb, xo, box, f);
                                else dequant_chunk_lanes_outl<true, false>(v, row_scale, ca, cb, xo, box, f);
                            } else {
                                if (uni) dequant_chunk_lanes_outl<false, true>(v, row_scale, ca, cb, xo, box, f);
                                else dequant_chunk_lanes_outl<false, false>(v, row_scale, ca, cb, xo, box, f);
                            }
                        } else if (gelu) {
                            if (uni) dequant_chunk_lanes<true, true>(v, row_scale, ca, cb, f);
                            else dequant_chunk_lanes<true, false>(v, row_scale, ca, cb, f);
                        } else {
                            if (uni) dequant_chunk_lanes<false, true>(v, row_scale, ca, cb, f);
                            else dequant_chunk_lanes<false, false>(v, row_scale, ca, cb, f);
                        }
                        if constexpr (EPI == EPI_BF16) {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float t0, t1;
                                f2_unpack(f[i], t0, t1);
                                w[i] = pack_bf16x2(t0, t1);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                float t0, t1;
                                f2_unpack(f[i], t0, t1);
                                w[2 * i] = __float_as_uint(t0);
                                w[2 * i + 1] = __float_as_uint(t1);
                                // columns past N carry zero factors, so they add 0
                                if (EPI == EPI_REQ && row_ok) amax = fmaxf(amax, fmaxf(fabsf(t0), fabsf(t1)));
                            }
                        }
                    }
                    if (lane == 0) bulk_wait_read_all();  // previous box of this warp has been read
                    __syncwarp();
                    stage_row_swizzled<RB>(stg, lane, w);
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmY, stg_s, n0, mt * BM + quarter * 32);
                        bulk_commit();
                    }
                }
                // accumulator b may be overwritten once every epilogue warp has read it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_tempty(b));
                if constexpr (EPI == EPI_REQ) {
                    if (row_ok) atomicMax(p.amax + gm, __float_as_uint(amax));
                }
            }
            if (lane == 0) bulk_wait_all();  // this warp's TMA stores have landed
        } else {
            float* st_a = stage_f;                  // per-column scale (or token scale when swapped)
            uint32_t lt = 0;
            for (int tile = cl; tile < num_tiles; tile += ncl, ++lt) {
                int mt, nt;
                tile_coords(tile, m_tiles, n_tiles, p.group_m, mt, nt);
                const int b = lt & 1;
                const uint32_t tph = (lt >> 1) & 1u;
                if constexpr (SWAP) {
                    if (S > 1 && rank > 0) {
                        // split-K helper: export this slice's partial accumulators to
                        // shared memory for the leader, once the leader has consumed
                        // the previous use of buffer b
                        const bool fr = mbar_wait(bar_red_free(b), tph ^ 1u, abort_flag, p.status, SITE_EPI_TMEM_FULL);
                        const bool tf = fr && mbar_wait(bar_tfull(b), tph, abort_flag, p.status, SITE_EPI_TMEM_FULL);
                        if (!named_bar_and(1, kEpiThreads, tf)) break;
                        tc_fence_after();
                        const uint32_t t_row = tmem_base + (uint32_t)(b * BN) + ((uint32_t)(quarter * 32) << 16);
                        int32_t* part = reinterpret_cast<int32_t*>(gbase + (sPart - base)) + (b * BM + r) * BN;
    #pragma unroll 1
                        for (int c = c_begin; c < c_end; ++c) {
                            uint32_t v[CW];
                            if constexpr (CW == 32) tmem_ld_32x32b_x32(t_row + c * CW, v);
                            else tmem_ld_32x32b_x16(t_row + c * CW, v);
                            tmem_ld_wait();
    #pragma unroll
                            for (int q4 = 0; q4 < CW / 4; ++q4)
                                reinterpret_cast<int4*>(part + c * CW)[q4] =
                                    make_int4((int)v[4 * q4], (int)v[4 * q4 + 1], (int)v[4 * q4 + 2], (int)v[4 * q4 + 3]);
                        }
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_tempty(b));
                        // every thread's partials are ordered before this CTA barrier;
                        // one cluster-scope fence by the arriving thread then
                        // releases them all to the leader (cumulativity)
                        named_bar_sync(1, kEpiThreads);
                        if (et == 0) {
                            fence_acq_rel_cluster();
                            mbar_arrive_cluster(mapa_shared(bar_red_full(b), 0u));
                        }
                        continue;
                    }
                }
                // stage the per-column factors of this tile (previous readers done)
                named_bar_sync(1, kEpiThreads);
                for (int i = et; EPI != EPI_I32 && i < BN; i += kEpiThreads) {
                    const int n = nt * BN + i;
                    const bool in = n < p.N;
                    st_a[i] = (EPI != EPI_I32 && in) ? __ldg(p.s_tok + n) : 0.0f;
                }
                named_bar_sync(1, kEpiThreads);
                // all 128 epilogue threads take the same decision (barrier with an
                // AND-reduction), so none is left behind at a later barrier
                bool got = mbar_wait(bar_tfull(b), tph, abort_flag, p.status, SITE_EPI_TMEM_FULL);
                if (SWAP && S > 1)  // split-K leader: the other slices' partials are in
                    got = got && mbar_wait_cluster(bar_red_full(b), tph, abort_flag, p.status, SITE_EPI_TMEM_FULL);
                if (!named_bar_and(1, kEpiThreads, got)) break;
                tc_fence_after();

                const int gm = mt * BM + r;          // M-side row owned by this thread
                const bool row_ok = gm < p.M;
                float row_scale = 0.0f, row_bias = 0.0f;
                if (EPI != EPI_I32 && row_ok) {
                    row_scale = __ldg(p.s_grp + gm / p.G);
                    row_bias = p.bias ? __ldg(p.bias + gm) : 0.0f;
                }
                const uint32_t t_row = tmem_base + (uint32_t)(b * BN) + ((uint32_t)(quarter * 32) << 16);
                static_assert(SWAP || CW == 32, "non-swapped tiles are whole 32-column chunks");

    #pragma unroll 1
                for (int c = c_begin; c < c_end; ++c) {
                    uint32_t v[CW];
                    if constexpr (CW == 32) tmem_ld_32x32b_x32(t_row + c * CW, v);
                    else tmem_ld_32x32b_x16(t_row + c * CW, v);
                    tmem_ld_wait();
                    if (SWAP && S > 1) {
                        // exact int32 sum of the K slices: peers' partials over DSMEM
                        const uint32_t own = sPart + (uint32_t)((b * BM + r) * BN + c * CW) * 4u;
                        for (int q = 1; q < S; ++q) {
                            const uint32_t src = mapa_shared(own, (uint32_t)q);
    #pragma unroll
                            for (int q4 = 0; q4 < CW / 4; ++q4) {
                                const int4 t4 = ld_cluster_v4(src + 16u * q4);
                                v[4 * q4] += (uint32_t)t4.x;
                                v[4 * q4 + 1] += (uint32_t)t4.y;
                                v[4 * q4 + 2] += (uint32_t)t4.z;
                                v[4 * q4 + 3] += (uint32_t)t4.w;
                            }
                        }
                    }
                    const int n0 = nt * BN + c * CW;   // first N-side index of the chunk
                    // thread owns output feature gm, columns = tokens n0 .. n0+CW-1
#pragma unroll
                    for (int j = 0; j < CW; ++j) {
                        const int tok = n0 + j;
                        float t = 0.0f;
                        if (EPI != EPI_I32) {
                            t = fmaf(row_scale * st_a[c * CW + j], (float)(int)v[j], row_bias);
                            if (p.act == ZQ_ACT_GELU) t = gelu_f(t);
                        }
                        if (EPI == EPI_REQ) {
                            // absmax over this warp's 32 features, one atomic per token
                            float m = (row_ok && tok < p.N) ? fabsf(t) : 0.0f;
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1)
                                m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                            if (lane == 0 && tok < p.N) atomicMax(p.amax + tok, __float_as_uint(m));
                        }
                        if (!row_ok || tok >= p.N) continue;
                        const int64_t off = (int64_t)tok * p.ldy + gm;
                        if constexpr (EPI == EPI_I32) static_cast<int32_t*>(p.y)[off] = (int32_t)v[j];
                        else if constexpr (EPI == EPI_BF16)
                            static_cast<__nv_bfloat16*>(p.y)[off] = __float2bfloat16_rn(t);
                        else static_cast<float*>(p.y)[off] = t;
                    }
                }
                // accumulator b may be overwritten once all four warps have read it
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_tempty(b));
                if (SWAP && S > 1) {
                    // the peers' partial buffers b have been read: hand them back
                    named_bar_sync(1, kEpiThreads);
                    if (et == 0)
                        for (int q = 1; q < S; ++q) mbar_arrive_cluster(mapa_shared(bar_red_free(b), (uint32_t)q));
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (SWAP) cluster_sync_all();  // no CTA leaves while a peer may still read its shared memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

// ------------------------------------------------------------ host side

constexpr int kMaxDevices = 64;

// Largest number of co-resident clusters of `S` CTAs for this kernel (cached).
template <typename K>
int max_clusters(K kern, int S, size_t smem, int threads, int dev) {
    static int cache[kMaxDevices][9] = {};
    if (S < 1 || S > 8) return 0;
    std::lock_guard<std::mutex> lk(launch_cache_mutex());
    if (cache[dev][S] == 0) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = S;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(S);
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
            cudaGetLastError();
            n = -1;
        }
        cache[dev][S] = n;
    }
    return cache[dev][S];
}

template <int BN, int STAGES, bool SWAP, int EPI, int EW, bool OUTL = false>
int launch_cfg(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, const Params& p,
               const DeviceInfo& di, cudaStream_t st) {
    constexpr size_t kSmem = smem_bytes<BN, STAGES, SWAP, EPI, EW>();
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(kSmem > 116 * 1024, "one CTA per SM (TMEM ownership)");
    auto kern = w8a8_gemm_kernel<BN, STAGES, SWAP, EPI, EW, OUTL>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    {
        std::lock_guard<std::mutex> lk(launch_cache_mutex());
        if (!attr_set[dev]) {
            int rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                      (int)kSmem));
            if (rc) return rc;
            attr_set[dev] = true;
        }
    }
    const int tiles = ((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
    if constexpr (SWAP) {
        // split K over a cluster of S CTAs: S minimising (rounds of tiles) / S,
        // with a small charge per extra slice; each slice keeps >= 1 k-block
        const int kblocks = (p.K + BK - 1) / BK;
        int bestS = 1, bestN = 0;
        double best = 1e30;
        for (int S = 1; S <= 8 && S <= kblocks; ++S) {
            const int n = max_clusters(kern, S, kSmem, block_threads<EW>(), dev);
            if (n < 1) continue;
            const int ncl = n < tiles ? n : tiles;
            const int rounds = (tiles + ncl - 1) / ncl;
            const double cost = (double)rounds / S + 0.03 * (S - 1);
            if (cost < best) {
                best = cost;
                bestS = S;
                bestN = ncl;
            }
        }
        if (bestN < 1) return ZQ_ERR_CUDA;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[2];
        at[0].id = cudaLaunchAttributeClusterDimension;
        at[0].val.clusterDim.x = bestS;
        at[0].val.clusterDim.y = 1;
        at[0].val.clusterDim.z = 1;
        cfg.attrs = at;
        cfg.numAttrs = 1 + (unsigned)pdl_attr(at[1]);
        cfg.gridDim = dim3(bestN * bestS);
        cfg.blockDim = dim3(block_threads<EW>());
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = st;
        count_launch();
        return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
    } else {
        const int grid = tiles < di.sm_count ? tiles : di.sm_count;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute at[1];
        cfg.attrs = at;
        cfg.numAttrs = (unsigned)pdl_attr(at[0]);
        cfg.gridDim = dim3((unsigned)grid);
        cfg.blockDim = dim3(block_threads<EW>());
        cfg.dynamicSmemBytes = kSmem;
        cfg.stream = st;
        count_launch();
        return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
    }
}

// Pipeline depth: as many stages as fit beside the output staging boxes.
template <int BN, bool SWAP, int EPI>
constexpr int stages_for() {
    if (SWAP) return BN == 64 ? 6 : 8;  // beside the split-K partial buffers
    if (BN == 256) return (EPI == EPI_BF16 || EPI == EPI_I32) ? 4 : 3;
    if (BN == 192) return 4;
    return 5;
}

template <int BN, bool SWAP>
int launch_epi(int epi, const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty,
               const Params& p, const DeviceInfo& di, cudaStream_t st) {
    // the epilogue is the long pole for short K loops: 16 warps (4 per SM
    // sub-partition) when it dequantizes, 8 for raw int32 and the decode shapes
    constexpr int EW = SWAP ? 8 : 16;
    switch (epi) {
        case EPI_I32: return launch_cfg<BN, stages_for<BN, SWAP, EPI_I32>(), SWAP, EPI_I32, 8>(ta, tb, ty, p, di, st);
        case EPI_F32: return launch_cfg<BN, stages_for<BN, SWAP, EPI_F32>(), SWAP, EPI_F32, EW>(ta, tb, ty, p, di, st);
        case EPI_BF16: return launch_cfg<BN, stages_for<BN, SWAP, EPI_BF16>(), SWAP, EPI_BF16, EW>(ta, tb, ty, p, di, st);
        default: return launch_cfg<BN, stages_for<BN, SWAP, EPI_REQ>(), SWAP, EPI_REQ, EW>(ta, tb, ty, p, di, st);
    }
}

// Tile width for the non-swapped kernel: every CTA runs whole tiles, so the
// time goes as (waves of tiles) x (tile width) / (efficiency of that width);
// narrower tiles re-read A more often and feed the MMA less per byte
// (measured on B200: 192 wide ~0.85, 128 wide ~0.7 of a 256-wide tile).
int pick_bn(int64_t T, int64_t N, int sms) {
    const int cands[3] = {256, 192, 128};
    const int64_t inv_eff_x20[3] = {20, 24, 29};  // 20 / efficiency
    int best = 256;
    int64_t best_cost = -1;
    const int64_t m_tiles = (T + BM - 1) / BM;
    for (int i = 0; i < 3; ++i) {
        const int bn = cands[i];
        const int64_t tiles = m_tiles * ((N + bn - 1) / bn);
        const int64_t waves = (tiles + sms - 1) / sms;
        const int64_t cost = waves * bn * inv_eff_x20[i];
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

}  // namespace

static PFN_cuTensorMapEncodeTiled_v12000 lookup_encode_fn() {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
}

// looked up once per process (a function-local static is initialised once,
// even when several threads make their first call together)
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = lookup_encode_fn();
    return fn;
}

int make_tmap_i8(CUtensorMap* tm, const void* ptr, int64_t rows, int64_t K, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return ZQ_ERR_CUDA;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ZQ_OK : ZQ_ERR_CUDA;
}


int make_tmap_out(CUtensorMap* tm, void* ptr, int64_t rows, int64_t cols, int esize) {
    auto fn = encode_fn();
    if (!fn) return ZQ_ERR_CUDA;
    const CUtensorMapDataType dt = esize == 1   ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                   : esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16
                                                : CU_TENSOR_MAP_DATA_TYPE_UINT32;
    const CUtensorMapSwizzle sw = esize == 1   ? CU_TENSOR_MAP_SWIZZLE_32B
                                  : esize == 2 ? CU_TENSOR_MAP_SWIZZLE_64B
                                               : CU_TENSOR_MAP_SWIZZLE_128B;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(cols * esize)};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(tm, dt, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? ZQ_OK : ZQ_ERR_CUDA;
}

int launch_w8a8_gemm(const LinearArgs& a, const DeviceInfo& di, cudaStream_t st) {
    int epi;
    switch (a.out_kind) {
        case ZQ_OUT_F32: epi = EPI_F32; break;
        case ZQ_OUT_BF16: epi = EPI_BF16; break;
        case ZQ_OUT_I8_REQUANT: epi = EPI_REQ; break;
        default: epi = EPI_I32; break;
    }
    Params p{};
    p.K = (int)a.K;
    p.G = (int)a.G;
    p.ldy = (int)a.N;
    p.s_tok = a.s_tok;
    p.s_grp = a.s_grp;
    p.bias = a.bias;
    p.y = epi == EPI_REQ ? static_cast<void*>(a.h_ws) : a.y;
    p.amax = a.amax_ws;
    p.act = a.act;
    p.status = di.status_word;
    p.group_m = (int)((a.N + BM - 1) / BM);  // swapped: plain row-tile-fastest order

    const bool swap = a.T <= 64;
    CUtensorMap ta, tb;
    int rc;
    if (swap) {
        // M side = weights [N, K]; N side = tokens [T, K], BN = T rounded up to 16 (<= 64)
        p.M = (int)a.N;
        p.N = (int)a.T;
        const int bn = a.T <= 16 ? 16 : a.T <= 32 ? 32 : 64;
        if ((rc = make_tmap_i8(&ta, a.Wq, a.N, a.K, BM))) return rc;
        if ((rc = make_tmap_i8(&tb, a.xq, a.T, a.K, bn))) return rc;
        // the transposed output is written directly (ty is not used)
        if (bn == 16) return launch_epi<16, true>(epi, ta, tb, ta, p, di, st);
        if (bn == 32) return launch_epi<32, true>(epi, ta, tb, ta, p, di, st);
        return launch_epi<64, true>(epi, ta, tb, ta, p, di, st);
    }
    p.M = (int)a.T;
    p.N = (int)a.N;
    const int bn = pick_bn(a.T, a.N, di.sm_count);
    {
        // row tiles per raster group: their activation slice (128 rows x K
        // bytes each) within ~24 MB of L2, at least one wave's worth of rows
        const int64_t m_tiles = (a.T + BM - 1) / BM;
        int64_t gm = (24ll << 20) / ((int64_t)BM * a.K);
        const int64_t n_tiles = (a.N + bn - 1) / bn;
        const int64_t min_gm = (di.sm_count + n_tiles - 1) / n_tiles;
        if (gm < min_gm) gm = min_gm;
        if (gm < 1) gm = 1;
        p.group_m = (int)(gm < m_tiles ? gm : m_tiles);
    }
    if ((rc = make_tmap_i8(&ta, a.xq, a.T, a.K, BM))) return rc;
    if ((rc = make_tmap_i8(&tb, a.Wq, a.N, a.K, bn))) return rc;
    CUtensorMap ty;
    if ((rc = make_tmap_out(&ty, p.y, a.T, a.N, epi == EPI_BF16 ? 2 : 4))) return rc;
    // stages: as many as fit beside the output staging boxes
    if (bn == 256) return launch_epi<256, false>(epi, ta, tb, ty, p, di, st);
    if (bn == 192) return launch_epi<192, false>(epi, ta, tb, ty, p, di, st);
    return launch_epi<128, false>(epi, ta, tb, ty, p, di, st);
}

// LLM.int8() linear: the W8A8 GEMM whose epilogue adds the fp16 outlier
// product before bias and activation (always the non-swapped kernel, 128-wide
// tiles; fp32 or bf16 output).
int launch_w8a8_gemm_outliers(const LinearArgs& a, const uint16_t* xo, const uint16_t* wo, const DeviceInfo& di,
                              cudaStream_t st) {
    const int epi = a.out_kind == ZQ_OUT_F32 ? EPI_F32 : EPI_BF16;
    Params p{};
    p.M = (int)a.T;
    p.N = (int)a.N;
    p.K = (int)a.K;
    p.G = (int)a.G;
    p.ldy = (int)a.N;
    p.s_tok = a.s_tok;
    p.s_grp = a.s_grp;
    p.bias = a.bias;
    p.y = a.y;
    p.act = a.act;
    p.status = di.status_word;
    p.xo = xo;
    p.wo = wo;
    const int64_t m_tiles = (a.T + BM - 1) / BM;
    int64_t gm = (24ll << 20) / ((int64_t)BM * a.K);
    const int64_t n_tiles = (a.N + 127) / 128;
    const int64_t min_gm = (di.sm_count + n_tiles - 1) / n_tiles;
    if (gm < min_gm) gm = min_gm;
    if (gm < 1) gm = 1;
    p.group_m = (int)(gm < m_tiles ? gm : m_tiles);
    CUtensorMap ta, tb, ty;
    int rc;
    if ((rc = make_tmap_i8(&ta, a.xq, a.T, a.K, BM))) return rc;
    if ((rc = make_tmap_i8(&tb, a.Wq, a.N, a.K, 128))) return rc;
    if ((rc = make_tmap_out(&ty, a.y, a.T, a.N, epi == EPI_BF16 ? 2 : 4))) return rc;
    if (epi == EPI_F32)
        return launch_cfg<128, stages_for<128, false, EPI_F32>(), false, EPI_F32, 16, true>(ta, tb, ty, p, di, st);
    return launch_cfg<128, stages_for<128, false, EPI_BF16>(), false, EPI_BF16, 16, true>(ta, tb, ty, p, di, st);
}

}  // namespace zq
