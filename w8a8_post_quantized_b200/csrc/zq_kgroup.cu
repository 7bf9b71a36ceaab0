// zq_kgroup.cu -- W8A8 linear with K-axis weight groups on sm_100a: one
// scale per output row and Gk consecutive input columns.  The scale now
// varies along the contraction, so each group's INT32 partial product is
// scaled on its own before the groups are summed.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (group-wise weight
// quantization; the pages' Ampere kernel sizes the group to the tensor-core
// tile) and "探秘Transformer系列之（36）— 大模型量化方案" §1.2.2 (group-wise
// weights; the INT32 accumulation scaled by the weight and activation
// scales), read along the input axis:
//   acc_j[t, o] = sum over k in group j of xq[t, k] * Wq[o, k]      (exact)
//   y[t, o]     = act(s_tok[t] * sum_j s_w[j, o] * acc_j[t, o] + bias[o])
// with s_w stored group-major ([K/Gk, N]) so one group's scales for a tile's
// columns are contiguous.
//
// Structure (one persistent CTA per SM, 128 x 128 tiles, 12 warps in three
// warpgroups; warpgroup 0 gives up registers to the epilogue with
// setmaxnreg: 40 per thread there, 232 in warpgroups 1-2):
//   warp 0   TMA producer: operand stages (128 rows x 128 bytes of each
//            operand, 128-byte swizzle);
//   warp 1   one thread issues tcgen05.mma kind::i8 (K = 32 each) into one of
//            NSLOT TMEM accumulators -- one accumulator per group -- and
//            commits the slot after the group's last k-step;
//   warps 2-3 idle;
//   warps 4-11 epilogue (two per TMEM lane quarter, 64 columns each): per
//            group, one tcgen05.ld round trip for the slot, each value scaled
//            by its column's group scale and added to fp32 running sums in
//            registers; after a tile's last group: token scale, bias,
//            optional GeLU, TMA store (fp32 or bf16).  Each warp fetches the
//            group scales of its own columns KG_PF groups ahead with
//            asynchronous 8-byte copies into a small ring in shared memory,
//            so neither the producer nor the MMA ever waits on them.
// The accumulator ring runs across tiles, so the MMAs of the next tile
// overlap the last groups and the output of the current one.
//
// Conversion without cvt: each slot holds the word 0x4B400000 (the fp32
// 1.5 * 2^23) before its first MMA and every MMA accumulates onto it, so the
// slot ends as the fp32 value 1.5 * 2^23 + acc_j, exact for |acc_j| <= 2^22
// (Gk <= 256: |acc_j| <= 128 * 128 * 256 = 2^22).  One packed subtraction
// recovers acc_j exactly and one packed FMA scales and accumulates it; the
// epilogue writes the word back after reading, ready for the slot's next
// group.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int KG_BM = 128;
constexpr int KG_BN = 128;
constexpr int KG_BK = 128;     // K bytes per stage (one swizzle row)
constexpr int KG_UK = 32;      // K per tcgen05.mma of kind::i8
constexpr int KG_NSLOT = 4;    // TMEM accumulators: 4 x 128 columns = all of TMEM
constexpr int KG_PF = 4;       // group scales fetched this many groups ahead
constexpr int KG_RING = KG_PF + 1;
constexpr int KG_EW = 8;                        // epilogue warps
constexpr int KG_THREADS = 128 + 32 * KG_EW;    // warpgroup 0 + two epilogue warpgroups
constexpr uint32_t KG_REG_LAUNCH = 168;         // registers per thread at launch (65536 / 384, rounded to 8)
constexpr uint32_t KG_REG_LOW = 40;             // warpgroup 0 after setmaxnreg.dec
constexpr uint32_t KG_REG_HIGH = 232;           // epilogue warpgroups after setmaxnreg.inc
static_assert(128 * KG_REG_LOW + 256 * KG_REG_HIGH <= KG_THREADS * KG_REG_LAUNCH,
              "the epilogue's registers come out of the block's launch allocation");
constexpr int KG_A = KG_BM * KG_BK;
constexpr int KG_B = KG_BN * KG_BK;
constexpr uint32_t kMagicBits = 0x4B400000u;  // 1.5 * 2^23
constexpr float kMagic = 12582912.0f;
enum { KG_F32 = 0, KG_BF16 = 1 };

enum KgSite {
    KG_SITE_PROD_EMPTY = 0x501,
    KG_SITE_MMA_FULL = 0x503,
    KG_SITE_MMA_SLOT = 0x504,
    KG_SITE_EPI_SLOT = 0x505,
    KG_SITE_DRAIN = 0x506,
};

struct KgParams {
    int M, N, K, G;       // tokens, outputs, reduction length, columns per group
    const float* s_tok;   // [M]
    const float* s_w;     // [K/G, N]
    const float* bias;    // [N] or null
    int act;
    int group_m;          // tile raster: groups of group_m row tiles sweep all column tiles
    int* status;
};

template <int EPI>
__host__ __device__ constexpr int kg_rb() { return EPI == KG_BF16 ? 64 : 128; }

template <int EPI, int EW, int STAGES>
__host__ __device__ constexpr size_t kg_smem() {
    // alignment slack + operand ring + one 32x32 output box per epilogue warp
    // + per-warp scale rings (KG_RING groups x the warp's columns) + barriers and flags
    return 1024 + (size_t)STAGES * (KG_A + KG_B) + (size_t)EW * 32 * kg_rb<EPI>() +
           (size_t)EW * KG_RING * (KG_BN / (EW / 4)) * 4 + 256;
}

// One 32-bit word into 32 lanes x 32 consecutive TMEM columns (the warp's
// lane quarter): the same register for every column.
__device__ __forceinline__ void tmem_st_splat_x32(uint32_t taddr, uint32_t w) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, "
        "%1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1, %1};" ::"r"(taddr),
        "r"(w)
        : "memory");
}

__device__ __forceinline__ void cp_async_8(uint32_t dst, const void* src, uint32_t src_bytes) {
    // src_bytes 0 fills the 8 bytes with zeros and reads nothing
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Tile index -> (row tile, column tile): groups of GM row tiles, row tile
// fastest inside a group, so the group's activation rows stay in L2 while the
// weight column tiles stream past.
__device__ __forceinline__ void kg_tile(int tile, int m_tiles, int n_tiles, int GM, int& mt, int& nt) {
    const int per_group = GM * n_tiles;
    const int g = tile / per_group;
    const int rem = tile - g * per_group;
    const int gm = min(GM, m_tiles - g * GM);
    mt = g * GM + rem % gm;
    nt = rem / gm;
}

template <int EPI, int EW, int STAGES>
__global__ void __launch_bounds__(KG_THREADS, 1)
w8a8_kgroup_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmY, const KgParams p) {
    static_assert(EW == KG_EW, "two epilogue warpgroups");
    constexpr int SLICES = EW / 4;
    constexpr int COLS = KG_BN / SLICES;  // columns per epilogue warp
    constexpr int NCH = COLS / 32;        // 32-column chunks per epilogue warp
    constexpr int RB = kg_rb<EPI>();
    constexpr uint32_t IDESC = idesc_i8(KG_BM, KG_BN);

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* gbase = smem_raw + (base - raw);
    const uint32_t sA = base;
    const uint32_t sB = sA + STAGES * KG_A;
    const uint32_t sStg = sB + STAGES * KG_B;
    const uint32_t sRing = sStg + (uint32_t)EW * 32u * RB;  // [EW][KG_RING][COLS] fp32
    const uint32_t sBar = sRing + (uint32_t)EW * KG_RING * COLS * 4u;
    uint8_t* gBar = gbase + (sBar - base);
    // barriers: full[S], empty[S], afull[NSLOT], (unused)[NSLOT], sempty[NSLOT], drain
    auto bar_full = [&](int s) { return sBar + 8u * s; };
    auto bar_empty = [&](int s) { return sBar + 8u * (STAGES + s); };
    auto bar_afull = [&](int s) { return sBar + 8u * (2 * STAGES + s); };               // accumulator done
    auto bar_sempty = [&](int s) { return sBar + 8u * (2 * STAGES + 2 * KG_NSLOT + s); };  // slot free
    const uint32_t bar_drain = sBar + 8u * (2 * STAGES + 3 * KG_NSLOT);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gBar + 8 * (2 * STAGES + 3 * KG_NSLOT + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int s = 0; s < KG_NSLOT; ++s) {
            mbar_init(bar_afull(s), 1);
            mbar_init(bar_sempty(s), EW);
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
        tmem_alloc(smem_u32(tmem_slot), KG_NSLOT * KG_BN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    griddep_launch_dependents();
    const uint32_t tmem_base = *tmem_slot;

    const int m_tiles = (p.M + KG_BM - 1) / KG_BM;
    const int n_tiles = (p.N + KG_BN - 1) / KG_BN;
    const int num_tiles = m_tiles * n_tiles;
    const int kblocks = (p.K + KG_BK - 1) / KG_BK;
    const int KS = p.K / KG_UK;     // k-steps (K is a multiple of G, G of 32)
    const int SPG = p.G / KG_UK;    // k-steps per group
    const int NG = p.K / p.G;       // groups per tile

    if (warp < 4) {
        // warpgroup 0 as a whole hands registers to the epilogue
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(KG_REG_LOW));
        if (warp == 0) {
            // ------------------------------------------------ TMA producer
            if (lane == 0) {
                griddep_wait();  // the activation codes are the previous grid's output
                uint32_t it = 0;
                bool ok = true;
                for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                    int mt, nt;
                    kg_tile(tile, m_tiles, n_tiles, p.group_m, mt, nt);
                    const int n0 = nt * KG_BN;
                    for (int kb = 0; kb < kblocks; ++kb) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait(bar_empty(s), ph ^ 1u, abort_flag, p.status, KG_SITE_PROD_EMPTY)) {
                            ok = false;
                            break;
                        }
                        mbar_arrive_expect_tx(bar_full(s), KG_A + KG_B);
                        tma_load_2d(sA + s * KG_A, &tmA, bar_full(s), kb * KG_BK, mt * KG_BM);
                        tma_load_2d(sB + s * KG_B, &tmB, bar_full(s), kb * KG_BK, n0);
                        ++it;
                    }
                }
                // every copy this thread issued lands before the CTA can exit
                const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
                for (uint32_t j = first; j < it; ++j)
                    mbar_wait(bar_full(j % STAGES), (j / STAGES) & 1u, nullptr, p.status, KG_SITE_DRAIN);
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                // One thread issues everything, so the loop keeps to counters (no
                // division): `left` = k-steps left in the current group.
                uint32_t it = 0, gc = 0, d = tmem_base;
                int left = 0;
                bool ok = true;
                // groups of whole 128-byte stages (every stage: 4 k-steps of one group)
                const bool aligned = SPG % 4 == 0 && p.K % KG_BK == 0;
                for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
                    for (int kb = 0; kb < kblocks; ++kb, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1u;
                        if (!mbar_wait(bar_full(s), ph, abort_flag, p.status, KG_SITE_MMA_FULL)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t da = sdesc_k_sw128(sA + s * KG_A);
                        const uint64_t db = sdesc_k_sw128(sB + s * KG_B);
                        const int nk = min(4, KS - 4 * kb);
                        if (aligned) {
                            // groups of whole stages: at most one group starts and
                            // one ends here, so the four MMAs issue back to back
                            if (left == 0) {
                                const uint32_t sl = gc & (KG_NSLOT - 1);
                                if (!mbar_wait(bar_sempty(sl), (gc / KG_NSLOT) & 1u, abort_flag, p.status,
                                               KG_SITE_MMA_SLOT)) {
                                    mma_commit(bar_empty(s));
                                    ok = false;
                                    break;
                                }
                                tc_fence_after();
                                d = tmem_base + sl * KG_BN;
                                left = SPG;
                            }
#pragma unroll
                            for (int k = 0; k < 4; ++k) mma_i8(d, da + 2u * k, db + 2u * k, IDESC, 1u);
                            left -= 4;
                            if (left == 0) {
                                mma_commit(bar_afull(gc & (KG_NSLOT - 1)));
                                ++gc;
                            }
                            mma_commit(bar_empty(s));  // stage free once these MMAs finish
                            continue;
                        }
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            if (k < nk && ok) {
                                if (left == 0) {
                                    // a new group: wait until its slot is drained and re-armed
                                    const uint32_t sl = gc & (KG_NSLOT - 1);
                                    if (!mbar_wait(bar_sempty(sl), (gc / KG_NSLOT) & 1u, abort_flag, p.status,
                                                   KG_SITE_MMA_SLOT)) {
                                        ok = false;
                                        break;
                                    }
                                    tc_fence_after();
                                    d = tmem_base + sl * KG_BN;
                                    left = SPG;
                                }
                                // +32 bytes along K inside the swizzle atom = +2 in the descriptor
                                mma_i8(d, da + 2u * k, db + 2u * k, IDESC, 1u);
                                if (--left == 0) {
                                    mma_commit(bar_afull(gc & (KG_NSLOT - 1)));
                                    ++gc;
                                }
                            }
                        }
                        mma_commit(bar_empty(s));  // stage free once these MMAs finish
                        if (!ok) break;
                    }
                }
                mma_commit(bar_drain);
                mbar_wait(bar_drain, 0u, nullptr, p.status, KG_SITE_DRAIN);
            }
            __syncwarp();
        }  // warps 2-3: idle
    } else {
        // ------------------------------------------------ epilogue
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(KG_REG_HIGH));
        griddep_wait();  // token scales come from the previous grid; y may still be read by it
        const int ew = warp - 4;
        const int quarter = warp & 3;      // TMEM lanes 32*quarter .. +31
        const int col0 = (ew >> 2) * COLS;  // this warp's columns of the tile
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint8_t* stg = gbase + (sStg - base) + (uint32_t)ew * 32u * RB;
        const uint32_t stg_s = smem_u32(stg);
        const bool gelu = p.act == ZQ_ACT_GELU;
        // arm every slot (the magic word in this warp's accumulator cells),
        // then release the slots once
        for (int sl = 0; sl < KG_NSLOT; ++sl)
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch)
                tmem_st_splat_x32(tmem_base + lane_off + (uint32_t)(sl * KG_BN + col0 + ch * 32), kMagicBits);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0)
            for (int sl = 0; sl < KG_NSLOT; ++sl) mbar_arrive(bar_sempty(sl));

        const uint64_t magic2 = f2_splat(kMagic);
        // this warp's scale ring: item i (the i-th group this warp handles,
        // tiles in order) lives in ring slot i % KG_RING; lane l fetches the
        // pair of columns 2l, 2l+1 (zeros past N)
        const uint32_t ring_s = sRing + (uint32_t)ew * KG_RING * COLS * 4u;
        const float* ring = reinterpret_cast<const float*>(gbase + (ring_s - base));
        // the prefetch cursor (tile, group, ring slot) advances by counters
        int pf_tile = blockIdx.x, pf_g = 0, pf_slot = 0;
        const float* pf_src = nullptr;  // this lane's scale pair in group 0 of pf_tile (null: past N)
        auto pf_tile_begin = [&]() {
            pf_src = nullptr;
            if (pf_tile < num_tiles) {
                int mt_, nt_;
                kg_tile(pf_tile, m_tiles, n_tiles, p.group_m, mt_, nt_);
                const int n = nt_ * KG_BN + col0 + 2 * lane;
                if (n < p.N) pf_src = p.s_w + n;  // N % 16 == 0: both columns or neither
            }
        };
        auto prefetch = [&]() {
            if (pf_tile < num_tiles)
                cp_async_8(ring_s + (uint32_t)(pf_slot * COLS + 2 * lane) * 4u,
                           pf_src ? pf_src + (size_t)pf_g * p.N : p.s_w, pf_src ? 8u : 0u);
            cp_async_commit();  // one group per item, empty past the end
            pf_slot = pf_slot == KG_RING - 1 ? 0 : pf_slot + 1;
            if (++pf_g == NG) {
                pf_g = 0;
                pf_tile += gridDim.x;
                pf_tile_begin();
            }
        };
        pf_tile_begin();
#pragma unroll
        for (int i = 0; i < KG_PF; ++i) prefetch();
        uint32_t gc = 0;  // item index
        int slot = 0;     // gc % KG_RING
        int prev_sl = -1;  // accumulator slot read last, released once its re-arm stores complete
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            int mt, nt;
            kg_tile(tile, m_tiles, n_tiles, p.group_m, mt, nt);
            const int gm = mt * KG_BM + r;
            const float row_scale = gm < p.M ? __ldg(p.s_tok + gm) : 0.0f;
            uint64_t run[NCH * 16];
#pragma unroll
            for (int i = 0; i < NCH * 16; ++i) run[i] = 0ull;  // +0.0f pairs
            bool alive = true;
            for (int g = 0; g < NG; ++g, ++gc) {
                const uint32_t sl = gc & (KG_NSLOT - 1);
                const uint32_t par = (gc / KG_NSLOT) & 1u;
                __syncwarp();  // every lane is done with the ring slot refilled next
                prefetch();    // item gc + KG_PF
                cp_async_wait<KG_PF>();  // this item's scales have landed (own lane) ...
                const bool got = mbar_wait(bar_afull(sl), par, abort_flag, p.status, KG_SITE_EPI_SLOT);
                if (!__all_sync(0xFFFFFFFFu, got)) {  // ... and every lane's (warp barrier)
                    alive = false;
                    break;
                }
                tc_fence_after();
                const uint32_t ta = tmem_base + lane_off + (uint32_t)(sl * KG_BN + col0);
                const float4* sc = reinterpret_cast<const float4*>(ring + slot * COLS);
                slot = slot == KG_RING - 1 ? 0 : slot + 1;
                // one TMEM round trip for all of this warp's columns
                uint32_t v[NCH][32];
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) tmem_ld_32x32b_x32(ta + ch * 32, v[ch]);
                tmem_ld_wait();
                // the previous slot's re-arm stores overlapped this slot's loads:
                // release it now
                if (prev_sl >= 0) {
                    tmem_st_wait();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_sempty(prev_sl));
                }
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch) tmem_st_splat_x32(ta + ch * 32, kMagicBits);  // re-arm
                prev_sl = (int)sl;
#pragma unroll
                for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 s4 = sc[ch * 8 + q];  // same address in every lane: a broadcast
                        const uint64_t a01 = f2_sub(u2_pack(v[ch][4 * q], v[ch][4 * q + 1]), magic2);
                        const uint64_t a23 = f2_sub(u2_pack(v[ch][4 * q + 2], v[ch][4 * q + 3]), magic2);
                        run[ch * 16 + 2 * q] = f2_fma(f2_pack(s4.x, s4.y), a01, run[ch * 16 + 2 * q]);
                        run[ch * 16 + 2 * q + 1] = f2_fma(f2_pack(s4.z, s4.w), a23, run[ch * 16 + 2 * q + 1]);
                    }
            }
            if (!alive) break;
            // y = act(s_tok * run + bias), one 32x32 box per chunk through a TMA store
            const uint64_t rs2 = f2_splat(row_scale);
#pragma unroll
            for (int ch = 0; ch < NCH; ++ch) {
                const int n0 = nt * KG_BN + col0 + ch * 32;
                uint32_t w[RB / 4];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    float4 b4 = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
                    if (p.bias && n0 + 4 * q < p.N) b4 = __ldg(reinterpret_cast<const float4*>(p.bias + n0) + q);
                    uint64_t f[2];
                    f[0] = f2_fma(rs2, run[ch * 16 + 2 * q], f2_pack(b4.x, b4.y));
                    f[1] = f2_fma(rs2, run[ch * 16 + 2 * q + 1], f2_pack(b4.z, b4.w));
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        if (gelu) f[h] = gelu2(f[h]);
                        float t0, t1;
                        f2_unpack(f[h], t0, t1);
                        const int i = 2 * q + h;
                        if constexpr (EPI == KG_BF16) {
                            w[i] = pack_bf16x2(t0, t1);
                        } else {
                            w[2 * i] = __float_as_uint(t0);
                            w[2 * i + 1] = __float_as_uint(t1);
                        }
                    }
                }
                if (lane == 0) bulk_wait_read_all();  // the previous box of this warp has been read
                __syncwarp();
                stage_row_swizzled<RB>(stg, lane, w);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmY, stg_s, n0, mt * KG_BM + quarter * 32);  // clipped at M and N
                    bulk_commit();
                }
            }
        }
        if (prev_sl >= 0) {  // release the last slot read
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_sempty(prev_sl));
        }
        cp_async_wait<0>();  // no scale copy outstanding at exit
        if (lane == 0) bulk_wait_all();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, KG_NSLOT * KG_BN);
    }
}

// Offline quantizer: one warp per group (row o, columns j*G .. j*G+G-1):
// absmax over the group, scale = absmax/127, codes rint(w * (127/absmax))
// clamped to [-127, 127]; the scale goes to s_w[j, o].
__global__ void __launch_bounds__(256)
kgroup_quant_kernel(const float* __restrict__ W, int64_t N, int64_t K, int G, int8_t* __restrict__ Wq,
                    float* __restrict__ s_w) {
    griddep_wait();  // writes weights: successors start only at completion
    const int lane = threadIdx.x & 31;
    const int64_t ng = K / G;
    const int64_t total = N * ng;
    const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t gid = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); gid < total; gid += nwarps) {
        const int64_t o = gid / ng, j = gid - o * ng;
        const float* src = W + o * K + j * G;
        int8_t* dst = Wq + o * K + j * G;
        float amax = 0.0f;
        for (int i = lane; i < G; i += 32) amax = fmaxf(amax, fabsf(__ldg(src + i)));
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o2));
        float scale, inv;
        absmax_scales(amax, scale, inv);
        for (int i = lane; i < G; i += 32) dst[i] = (int8_t)quant_code(__ldg(src + i), inv);
        if (lane == 0) s_w[j * N + o] = scale;
    }
}

constexpr int kMaxDevices = 64;

template <int EPI, int EW, int STAGES>
int kg_launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& ty, const KgParams& p,
              const DeviceInfo& di, cudaStream_t st) {
    constexpr size_t kSmem = kg_smem<EPI, EW, STAGES>();
    static_assert(kSmem <= 232448, "shared memory budget");
    static_assert(kSmem > 116 * 1024, "one CTA per SM (it owns all of TMEM)");
    auto kern = w8a8_kgroup_kernel<EPI, EW, STAGES>;
    static bool attr_set[kMaxDevices] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= kMaxDevices) return ZQ_ERR_DEVICE;
    std::unique_lock<std::mutex> lk(launch_cache_mutex());
    if (!attr_set[dev]) {
        int rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
        if (rc) return rc;
        attr_set[dev] = true;
    }
    // setmaxnreg.inc waits until the registers it asks for are free, so the
    // split must fit the registers the block is launched with
    static int launch_regs[kMaxDevices] = {};
    if (!launch_regs[dev]) {
        cudaFuncAttributes fa;
        int rc = cuda_status(cudaFuncGetAttributes(&fa, kern));
        if (rc) return rc;
        launch_regs[dev] = fa.numRegs;
    }
    const int regs = launch_regs[dev];
    lk.unlock();
    if ((uint32_t)regs * KG_THREADS < 128 * KG_REG_LOW + 256 * KG_REG_HIGH) {
        set_cuda_error(cudaErrorInvalidConfiguration);
        return ZQ_ERR_CUDA;
    }
    const int tiles = ((p.M + KG_BM - 1) / KG_BM) * ((p.N + KG_BN - 1) / KG_BN);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3((unsigned)(tiles < di.sm_count ? tiles : di.sm_count));
    cfg.blockDim = dim3(KG_THREADS);
    cfg.dynamicSmemBytes = kSmem;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, ty, p));
}

inline bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) % a) == 0; }

}  // namespace
}  // namespace zq

using namespace zq;

extern "C" {

int zq_quantize_weights_kgroups(const float* W, int64_t N, int64_t K, int64_t group_cols, int8_t* Wq, float* s_w,
                                void* stream) {
    if (!W || !Wq || !s_w) return ZQ_ERR_NULL;
    if (N <= 0 || K <= 0 || group_cols <= 0 || K % 16 != 0 || K % group_cols != 0 || group_cols > (1 << 30))
        return ZQ_ERR_SHAPE;
    if (N > ((int64_t)1 << 40) / K) return ZQ_ERR_SHAPE;
    if (!aligned(W, 16) || !aligned(Wq, 16) || !aligned(s_w, 4)) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    const int64_t warps = N * (K / group_cols);
    int64_t blocks = (warps + 7) / 8;
    if (blocks > (int64_t)di.sm_count * 16) blocks = (int64_t)di.sm_count * 16;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = static_cast<cudaStream_t>(stream);
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kgroup_quant_kernel, W, N, K, (int)group_cols, Wq, s_w));
}

int zq_w8a8_linear_kgroups(const int8_t* xq, const float* s_tok, int64_t T, int64_t K, const int8_t* Wq,
                           const float* s_w, int64_t N, int64_t group_cols, const float* bias, int act, int out_kind,
                           void* y, void* stream) {
    if (!xq || !s_tok || !Wq || !s_w || !y) return ZQ_ERR_NULL;
    if (out_kind != ZQ_OUT_F32 && out_kind != ZQ_OUT_BF16) return ZQ_ERR_DTYPE;
    if (act != ZQ_ACT_NONE && act != ZQ_ACT_GELU) return ZQ_ERR_DTYPE;
    if (T <= 0 || K <= 0 || N <= 0 || group_cols <= 0) return ZQ_ERR_SHAPE;
    if (group_cols % 32 != 0 || group_cols > 256 || K % group_cols != 0 || N % 16 != 0) return ZQ_ERR_SHAPE;
    if (T > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return ZQ_ERR_SHAPE;
    if (!aligned(xq, 16) || !aligned(Wq, 16) || !aligned(y, 16) || !aligned(s_w, 16) || !aligned(s_tok, 4))
        return ZQ_ERR_ALIGN;
    if (bias && !aligned(bias, 16)) return ZQ_ERR_ALIGN;
    DeviceInfo di;
    int rc = device_info(&di);
    if (rc) return rc;
    KgParams p{};
    p.M = (int)T;
    p.N = (int)N;
    p.K = (int)K;
    p.G = (int)group_cols;
    p.s_tok = s_tok;
    p.s_w = s_w;
    p.bias = bias;
    p.act = act;
    p.status = di.status_word;
    {
        // row tiles per raster group: their activation rows within ~24 MB of
        // L2, at least one wave's worth of tiles
        const int64_t m_tiles = (T + KG_BM - 1) / KG_BM;
        const int64_t n_tiles = (N + KG_BN - 1) / KG_BN;
        int64_t gm = (24ll << 20) / ((int64_t)KG_BM * K);
        const int64_t min_gm = (di.sm_count + n_tiles - 1) / n_tiles;
        if (gm < min_gm) gm = min_gm;
        if (gm < 1) gm = 1;
        p.group_m = (int)(gm < m_tiles ? gm : m_tiles);
    }
    CUtensorMap ta, tb, ty;
    if ((rc = make_tmap_i8(&ta, xq, T, K, KG_BM))) return rc;
    if ((rc = make_tmap_i8(&tb, Wq, N, K, KG_BN))) return rc;
    if ((rc = make_tmap_out(&ty, y, T, N, out_kind == ZQ_OUT_BF16 ? 2 : 4))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    if (out_kind == ZQ_OUT_BF16) return kg_launch<KG_BF16, 8, 6>(ta, tb, ty, p, di, st);
    return kg_launch<KG_F32, 8, 5>(ta, tb, ty, p, di, st);
}

}  // extern "C"
