// zq_rowquant.cu -- pipelined per-token quantizers for sm_100a:
// fused LayerNorm + quantize and fused (bias +) GeLU + quantize.
//
// Sources: "[2022 NeurIPS] ZeroQuant: Efficient and Affordable Post-Training
// Quantization for Large-Scale Transformers" (token-wise quantization fused
// with the preceding element-wise or reduction op: "LN/GeLU + Quantize") and
// "探秘Transformer系列之（36）— 大模型量化方案" §1.1.2 (absmax rule into
// [-127, 127]) and §1.2.2 (one dynamic scale per token, computed at run
// time, the quantizer fused with LayerNorm).
//
// HBM-bound: each input byte is read once and each code written once.  One
// persistent CTA per SM takes a contiguous range of rows.  Rows are processed
// by teams of TPR threads (half a warp for short rows, up to the whole CTA for
// long ones); each thread holds PPT pieces of the row in registers (a piece
// is 16 input bytes: 8 bf16 or 4 fp32 values, read from shared memory without
// bank conflicts), so the statistics need no second pass over memory.  Every
// row arrives by one 1-D bulk async copy into a shared-memory slot owned by
// its team; the team requests its next row into the slot as soon as the row
// it held is in registers, so each team keeps its other slots in flight while
// it computes.
#include "zq_internal.cuh"

namespace zq {
namespace {

constexpr int kSiteRowqFull = 0x401;
constexpr int kRingBytes = 220 * 1024;      // parameters + row slots, per CTA
constexpr int kMaxSlots = 128;              // one full barrier per slot (8 bytes each)
constexpr int kRedOffset = 8 * kMaxSlots;   // team reduction slots after the barriers
constexpr int kRingOffset = kRedOffset + 512;

// A piece is 16 input bytes held as NP packed fp32 pairs.
template <typename Tin>
struct Piece;

template <>
struct Piece<uint16_t> {  // bf16 bit patterns: 8 values, 4 pairs
    static constexpr int EPP = 8;
    static constexpr int NP = 4;
    static __device__ __forceinline__ void load(const uint16_t* p, uint64_t (&v)[NP]) {
        const uint4 a = *reinterpret_cast<const uint4*>(p);
        v[0] = f2_pack(bf16_lo(a.x), bf16_hi(a.x));
        v[1] = f2_pack(bf16_lo(a.y), bf16_hi(a.y));
        v[2] = f2_pack(bf16_lo(a.z), bf16_hi(a.z));
        v[3] = f2_pack(bf16_lo(a.w), bf16_hi(a.w));
    }
};

template <>
struct Piece<float> {  // 4 values, 2 pairs
    static constexpr int EPP = 4;
    static constexpr int NP = 2;
    static __device__ __forceinline__ void load(const float* p, uint64_t (&v)[NP]) {
        const ulonglong2 a = *reinterpret_cast<const ulonglong2*>(p);
        v[0] = a.x;
        v[1] = a.y;
    }
};

// NP pairs of fp32 parameters (gamma, beta or bias) of piece p.  A piece's
// parameters are NP/2 16-byte quarters.  In global memory they are
// contiguous; the shared-memory copy stores quarter h of every piece together
// (index h*nP + p), so the 16-byte loads of consecutive threads are
// contiguous and free of bank conflicts.
template <int NP, bool SMEM>
__device__ __forceinline__ void load_param_pairs(const float* base, int p, int nP, uint64_t (&v)[NP]) {
#pragma unroll
    for (int h = 0; h < NP / 2; ++h) {
        const ulonglong2* src =
            reinterpret_cast<const ulonglong2*>(SMEM ? base + ((size_t)h * nP + p) * 4 : base + (size_t)p * 2 * NP + h * 4);
        const ulonglong2 a = SMEM ? *src : __ldg(src);
        v[2 * h] = a.x;
        v[2 * h + 1] = a.y;
    }
}

__device__ __forceinline__ float f2_hsum(uint64_t v) {
    float a, b;
    f2_unpack(v, a, b);
    return a + b;
}

__device__ __forceinline__ float f2_absmax(float m, uint64_t v) {
    float a, b;
    f2_unpack(v, a, b);
    return fmaxf(m, fmaxf(fabsf(a), fabsf(b)));
}

// Reductions over the TPR threads of one team: xor shuffles inside a warp;
// for teams of several warps the warps' partials go to shared memory, the
// team's first warp merges them with shuffles and broadcasts the result
// (every thread merging all partials itself cost about three instructions per
// element at 12288-wide rows).  Teams smaller than the CTA use their own named
// barrier (id 1 + team) and their own words of `red`, so no two teams ever
// share a word (teams progress independently).
template <int TPR, int BLOCK>
struct Team {
    static constexpr int W = TPR > 32 ? TPR / 32 : 1;   // warps per team
    static constexpr int TEAMS = BLOCK / TPR;
    // words per team: statistics (n, mean, M2 per warp + the merged mean, M2)
    // and maxima (one per warp + the result)
    static constexpr int kStatWords = 3 * W + 2;
    static constexpr int kMaxWords = W + 1;
    static constexpr int kWords = TPR > 32 ? TEAMS * (kStatWords + kMaxWords) : 0;  // single-warp teams: none
    static __device__ __forceinline__ void sync(int team) {
        if constexpr (TPR == BLOCK) __syncthreads();
        else named_bar_sync(1 + team, TPR);
    }
    // xor-shuffle offsets stay inside a team when TPR < 32 (two teams per warp)
    static constexpr int kTopLane = TPR < 32 ? TPR / 2 : 16;

    // One merge step of per-thread (count, mean, sum of squared deviations)
    // with the partner `o` lanes away (Chan's pairwise update).  EQ: both
    // halves hold the same count n, so mean = (mean_a + mean_b) / 2 and
    // M2 = M2_a + M2_b + d^2 n / 2, no division.
    template <bool EQ>
    static __device__ __forceinline__ void merge_xor(float& n, float& mean, float& m2, int o) {
        const float mb = __shfl_xor_sync(0xFFFFFFFFu, mean, o);
        const float qb = __shfl_xor_sync(0xFFFFFFFFu, m2, o);
        if constexpr (EQ) {
            const float d = mb - mean;
            mean = fmaf(0.5f, d, mean);
            m2 = m2 + qb + d * d * (0.5f * n);
            n = n + n;
        } else {
            const float nb = __shfl_xor_sync(0xFFFFFFFFu, n, o);
            const float nt = n + nb;
            if (nt > 0.0f) {
                const float d = mb - mean;
                const float f = __fdividef(nb, nt);
                mean = fmaf(d, f, mean);
                m2 = m2 + qb + d * d * n * f;
                n = nt;
            }
        }
    }
    // The team's mean and M2 from every thread's (count, mean, M2).
    template <bool EQ = false>
    static __device__ __forceinline__ void stats(float n, float mean, float m2, float* red, int team,
                                                 float& mean_out, float& m2_out) {
#pragma unroll
        for (int o = kTopLane; o > 0; o >>= 1) merge_xor<EQ>(n, mean, m2, o);
        if constexpr (TPR > 32) {
            float* slot = red + team * kStatWords;
            const int w = (threadIdx.x % TPR) >> 5;
            const int lane = threadIdx.x & 31;
            if (lane == 0) {
                slot[3 * w] = n;
                slot[3 * w + 1] = mean;
                slot[3 * w + 2] = m2;
            }
            sync(team);
            if (w == 0) {
                // lanes 0..W-1 hold the warps' partials; xor offsets below W
                // keep them among themselves (W is a power of two)
                float nn = lane < W ? slot[3 * lane] : 0.0f;
                float mm = lane < W ? slot[3 * lane + 1] : 0.0f;
                float qq = lane < W ? slot[3 * lane + 2] : 0.0f;
#pragma unroll
                for (int o = W / 2; o > 0; o >>= 1) merge_xor<EQ>(nn, mm, qq, o);
                if (lane == 0) {
                    slot[3 * W] = mm;
                    slot[3 * W + 1] = qq;
                }
            }
            sync(team);
            mean = slot[3 * W];
            m2 = slot[3 * W + 1];
        }
        mean_out = mean;
        m2_out = m2;
    }
    // The team's maximum of non-negative values.
    static __device__ __forceinline__ float max(float v, float* red, int team) {
#pragma unroll
        for (int o = kTopLane; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if constexpr (TPR <= 32) {
            return v;
        } else {
            float* slot = red + TEAMS * kStatWords + team * kMaxWords;
            const int w = (threadIdx.x % TPR) >> 5;
            const int lane = threadIdx.x & 31;
            if (lane == 0) slot[w] = v;
            sync(team);
            if (w == 0) {
                float m = lane < W ? slot[lane] : 0.0f;
#pragma unroll
                for (int o = W / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
                if (lane == 0) slot[W] = m;
            }
            sync(team);
            return slot[W];
        }
    }
};

// Codes of one piece: computed by every thread, stored only where `store`
// (a predicated store, no branch around the arithmetic).
template <int NP, bool FUSED>
__device__ __forceinline__ void store_piece_codes_if(bool store, int8_t* dst, const uint64_t (&y)[NP],
                                                     uint64_t inv2) {
    if constexpr (NP == 4) {
        uint2 o;
        o.x = FUSED ? quant4_packed_fused(y[0], y[1], inv2) : quant4_packed(y[0], y[1], inv2);
        o.y = FUSED ? quant4_packed_fused(y[2], y[3], inv2) : quant4_packed(y[2], y[3], inv2);
        if (store) __stcs(reinterpret_cast<uint2*>(dst), o);
    } else {
        const uint32_t o = FUSED ? quant4_packed_fused(y[0], y[1], inv2) : quant4_packed(y[0], y[1], inv2);
        if (store) __stcs(reinterpret_cast<uint32_t*>(dst), o);
    }
}

// FULL: the row is exactly TPR * PPT pieces, so every piece of a row exists
// and the per-piece guards vanish at compile time.
//
// Rows: CTA b takes the contiguous rows [b * rows_per_cta, ...); within them
// team j takes local rows j, j + TEAMS, j + 2 TEAMS, ...  Each row is one
// 1-D bulk copy into a shared-memory slot; team j owns the per_team slots
// j, j + TEAMS, ..., and its i-th row uses slot j + (i % per_team) TEAMS in
// phase (i / per_team) & 1, so a team cycles through its own slots in row
// order and never waits on a slot more than one phase ahead.  As soon as the
// whole team holds a row in registers (after its first reduction) the team's
// leader refills the slot with the team's row per_team places later, so the
// team's other slots keep streaming while it computes.
template <typename Tin, bool LN, int TPR, int PPT, int BLOCK, bool SMEMP, bool FULL>
__global__ void __launch_bounds__(BLOCK, 1)
rowq_pipe_kernel(const Tin* __restrict__ x, int T, int H, float inv_h, int rows_per_cta, int per_team,
                 const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                 const float* __restrict__ bias, int act, int8_t* __restrict__ q,
                 float* __restrict__ s_tok, int* status) {
    constexpr int EPP = Piece<Tin>::EPP;
    constexpr int NP = Piece<Tin>::NP;
    constexpr int TEAMS = BLOCK / TPR;
    constexpr int TPW = TPR < 32 ? 32 / TPR : 1;   // teams per warp
    using TM = Team<TPR, BLOCK>;
    static_assert(TM::kWords * sizeof(float) <= kRingOffset - kRedOffset, "team reduction words");
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t bar0 = smem_u32(smem);          // full barrier of slot s at bar0 + 8 s
    float* red = reinterpret_cast<float*>(smem + kRedOffset);
    __shared__ int abort_flag;
    // per-column parameters (gamma and beta, or bias) copied once per CTA
    const int n_par = LN ? 2 : (bias ? 1 : 0);
    float* spar = reinterpret_cast<float*>(smem + kRingOffset);
    uint8_t* ring = smem + kRingOffset + (SMEMP ? (size_t)n_par * H * sizeof(float) : 0);
    const int row_bytes = H * (int)sizeof(Tin);
    const int nP = FULL ? TPR * PPT : H / EPP;  // pieces per row (compile-time when exact)
    const int team = threadIdx.x / TPR;
    const int tt = threadIdx.x % TPR;
    const int nslots = per_team * TEAMS;
    const int64_t r0 = (int64_t)blockIdx.x * rows_per_cta;
    const int n_local = (int)min((int64_t)rows_per_cta, (int64_t)T - r0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < nslots; ++s) mbar_init(bar0 + 8u * s, 1);
        abort_flag = 0;
        fence_proxy_async_smem();
        fence_barrier_init();
    }
    __syncthreads();
    griddep_wait();  // inputs and outputs are free of the previous grid in the stream
    griddep_launch_dependents();

    int last_issued = -1;  // the leader's latest request (its team's rows are requested in order)
    auto issue = [&](int li, int s) {
        last_issued = li;
        mbar_arrive_expect_tx(bar0 + 8u * s, (uint32_t)row_bytes);
        bulk_load(smem_u32(ring + (size_t)s * row_bytes), x + (r0 + li) * H, (uint32_t)row_bytes, bar0 + 8u * s);
    };
    // each team's leader requests the team's first rows before the parameters
    // are staged, so the two global-memory latencies overlap
    const bool leader = tt == 0;
    if (leader)
        for (int k = 0; k < per_team && team + k * TEAMS < n_local; ++k) issue(team + k * TEAMS, team + k * TEAMS);
    if constexpr (SMEMP) {
        const float* src0 = LN ? gamma : bias;
        constexpr int QPP = NP / 2;  // 16-byte quarters per piece
        for (int i = threadIdx.x; i < H / 4; i += BLOCK) {
            const int dst = (i % QPP) * nP + i / QPP;
            if (n_par >= 1) reinterpret_cast<float4*>(spar)[dst] = __ldg(reinterpret_cast<const float4*>(src0) + i);
            if (n_par == 2) reinterpret_cast<float4*>(spar + H)[dst] = __ldg(reinterpret_cast<const float4*>(beta) + i);
        }
    }
    const float* pg = SMEMP ? spar : gamma;
    const float* pb = SMEMP ? spar + H : beta;
    const float* pbias = SMEMP ? spar : bias;
    __syncthreads();

    // all teams sharing a warp run the same number of iterations (their
    // shuffles use the full warp); a team past the last row computes on a
    // stale slot, waits on nothing and stores nothing
    int ks = 0;            // slot index within the team: this row uses slot team + ks * TEAMS
    uint32_t phase = 0;    // parity of the slot's phase for this row
    for (int lb = team - team % TPW; lb < n_local; lb += TEAMS) {
        const int li = lb + team % TPW;
        const bool row_ok = li < n_local;
        const int s = team + ks * TEAMS;
        bool ok = !row_ok || mbar_wait(bar0 + 8u * s, phase, &abort_flag, status, kSiteRowqFull);
        ok = ok && !abort_flag;                     // a copy that never landed stops the whole CTA
        const bool use = row_ok && ok;
        const Tin* xr = reinterpret_cast<const Tin*>(ring + (size_t)s * row_bytes);
        const int64_t row = r0 + li;
        uint64_t v[PPT][NP];
        bool okp[PPT];
#pragma unroll
        for (int k = 0; k < PPT; ++k) {
            const int p = k * TPR + tt;
            okp[k] = use && (FULL || p < nP);
            if (FULL || okp[k]) Piece<Tin>::load(xr + p * EPP, v[k]);   // exact fit: always in the slot
            else {
#pragma unroll
                for (int i = 0; i < NP; ++i) v[k][i] = 0ull;
            }
        }
        // the team's row is in registers once its first reduction is done:
        // then the leader refills the slot (sub-warp teams: the warp's
        // shuffles and this __syncwarp order every lane's reads before it)
        auto refill = [&]() {
            if constexpr (TPR <= 32) __syncwarp();
            if (leader && use && li + nslots < n_local) issue(li + nslots, s);
        };
        float amax = 0.0f;
        if constexpr (LN) {
            // per-thread mean and squared deviations (two passes over the
            // registers, four independent accumulators each), merged over
            // the team
            uint64_t sa[4] = {0ull, 0ull, 0ull, 0ull};
            int nv = 0;
#pragma unroll
            for (int k = 0; k < PPT; ++k) {
                nv += (FULL || okp[k]) ? EPP : 0;
#pragma unroll
                for (int i = 0; i < NP; ++i) sa[(k * NP + i) & 3] = f2_add(sa[(k * NP + i) & 3], v[k][i]);
            }
            const float n_loc = FULL ? (float)(PPT * EPP) : (float)nv;
            const float sum_loc = f2_hsum(f2_add(f2_add(sa[0], sa[1]), f2_add(sa[2], sa[3])));
            const float mean_loc = FULL ? sum_loc * (1.0f / (float)(PPT * EPP))
                                        : (nv ? sum_loc * __frcp_rn(n_loc) : 0.0f);
            const uint64_t ml2 = f2_pack(mean_loc, mean_loc);
            uint64_t da[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                if (FULL || okp[k]) {
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        const uint64_t d = f2_sub(v[k][i], ml2);
                        da[(k * NP + i) & 3] = f2_fma(d, d, da[(k * NP + i) & 3]);
                    }
                }
            float mean, m2;
            TM::template stats<FULL>(n_loc, mean_loc,
                                     f2_hsum(f2_add(f2_add(da[0], da[1]), f2_add(da[2], da[3]))), red, team,
                                     mean, m2);
            refill();
            const float rstd = rsqrtf(fmaf(m2, inv_h, eps));
            const uint64_t mean2 = f2_pack(mean, mean);
            const uint64_t rstd2 = f2_pack(rstd, rstd);
            float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                if (FULL || okp[k]) {
                    const int p = k * TPR + tt;
                    uint64_t g[NP], b[NP];
                    load_param_pairs<NP, SMEMP>(pg, p, nP, g);
                    load_param_pairs<NP, SMEMP>(pb, p, nP, b);
#pragma unroll
                    for (int i = 0; i < NP; ++i) {
                        const uint64_t a = f2_mul(rstd2, g[i]);
                        const uint64_t y = f2_fma(f2_sub(v[k][i], mean2), a, b[i]);
                        v[k][i] = y;
                        am[(k * NP + i) & 3] = f2_absmax(am[(k * NP + i) & 3], y);
                    }
                }
            amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
            amax = TM::max(amax, red, team);
        } else {
            float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                if (FULL || okp[k]) {
                    if (bias) {
                        uint64_t b[NP];
                        load_param_pairs<NP, SMEMP>(pbias, k * TPR + tt, nP, b);
#pragma unroll
                        for (int i = 0; i < NP; ++i) v[k][i] = f2_add(v[k][i], b[i]);
                    }
                    if (act == ZQ_ACT_GELU) {
#pragma unroll
                        for (int i = 0; i < NP; ++i) {
                            float lo, hi;
                            f2_unpack(v[k][i], lo, hi);
                            v[k][i] = f2_pack(gelu_f(lo), gelu_f(hi));
                        }
                    }
#pragma unroll
                    for (int i = 0; i < NP; ++i) am[(k * NP + i) & 3] = f2_absmax(am[(k * NP + i) & 3], v[k][i]);
                }
            amax = fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3]));
            amax = TM::max(amax, red, team);
            refill();
        }
        // inv = 127/amax for every thread; scale = amax/127 only where it is stored
        const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
        const uint64_t inv2 = f2_pack(inv, inv);
        int8_t* qr = q + row * H;
        if (LN || act == ZQ_ACT_GELU) {
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                store_piece_codes_if<NP, true>(okp[k], qr + (k * TPR + tt) * EPP, v[k], inv2);
        } else {
#pragma unroll
            for (int k = 0; k < PPT; ++k)
                store_piece_codes_if<NP, false>(okp[k], qr + (k * TPR + tt) * EPP, v[k], inv2);
        }
        if (use && tt == 0) s_tok[row] = __fdiv_rn(amax, 127.0f);
        if (++ks == per_team) {
            ks = 0;
            phase ^= 1u;
        }
    }
    // no copy is left in flight when the CTA exits: every requested row was
    // waited for above unless a wait gave up; then the leader waits (bounded)
    // for its team's requests that may still be outstanding (the last
    // per_team of them)
    if (leader && abort_flag && last_issued >= 0)
        for (int li = max(team, last_issued - (per_team - 1) * TEAMS); li <= last_issued; li += TEAMS)
            mbar_wait(bar0 + 8u * (li % nslots), (uint32_t)(li / nslots) & 1u, nullptr, status, kSiteRowqFull);
}

template <typename Tin, bool LN>
using PipeKernel = void (*)(const Tin*, int, int, float, int, int, const float*, const float*, float,
                            const float*, int, int8_t*, float*, int*);

// (TPR, PPT, BLOCK) shapes: a team of TPR threads covers TPR*PPT pieces.
struct Shape {
    int tpr, ppt, block;
};
// Each thread holds 6-8 pieces (48-64 values) so the per-row costs
// (reductions, divisions) are spread over many elements, with 16 warps per SM.
// Teams are half a warp for short rows (two rows per warp, no barriers), one
// or more warps for longer rows.
constexpr Shape kShapes[] = {{16, 1, 512},   {16, 2, 512},  {16, 4, 512},  {16, 6, 512},
                             {16, 8, 512},   {32, 8, 512},  {64, 8, 512},  {128, 6, 512},
                             {128, 8, 512},  {256, 6, 512}, {256, 8, 512}, {256, 16, 256}};
constexpr int kNumShapes = 12;
constexpr int kFirstGlobalParamShape = 10;  // from here on parameters stay in global memory

template <typename Tin, bool LN, bool FULL>
PipeKernel<Tin, LN> pipe_kernel_t(int idx) {
    switch (idx) {
        case 0: return rowq_pipe_kernel<Tin, LN, 16, 1, 512, true, FULL>;
        case 1: return rowq_pipe_kernel<Tin, LN, 16, 2, 512, true, FULL>;
        case 2: return rowq_pipe_kernel<Tin, LN, 16, 4, 512, true, FULL>;
        case 3: return rowq_pipe_kernel<Tin, LN, 16, 6, 512, true, FULL>;
        case 4: return rowq_pipe_kernel<Tin, LN, 16, 8, 512, true, FULL>;
        case 5: return rowq_pipe_kernel<Tin, LN, 32, 8, 512, true, FULL>;
        case 6: return rowq_pipe_kernel<Tin, LN, 64, 8, 512, true, FULL>;
        case 7: return rowq_pipe_kernel<Tin, LN, 128, 6, 512, true, FULL>;
        case 8: return rowq_pipe_kernel<Tin, LN, 128, 8, 512, true, FULL>;
        case 9: return rowq_pipe_kernel<Tin, LN, 256, 6, 512, true, FULL>;
        case 10: return rowq_pipe_kernel<Tin, LN, 256, 8, 512, false, false>;
        default: return rowq_pipe_kernel<Tin, LN, 256, 16, 256, false, false>;
    }
}

// The kernel for shape idx; full: the row is exactly the shape's TPR * PPT pieces.
template <typename Tin, bool LN>
PipeKernel<Tin, LN> pipe_kernel(int idx, bool full) {
    return full ? pipe_kernel_t<Tin, LN, true>(idx) : pipe_kernel_t<Tin, LN, false>(idx);
}

// Smallest shape whose team covers the row's pieces.
int pick_shape(int pieces) {
    for (int i = 0; i < kNumShapes; ++i)
        if (kShapes[i].tpr * kShapes[i].ppt >= pieces) return i;
    return -1;
}

template <typename Tin, bool LN>
int launch_typed(const Tin* x, int64_t T, int64_t H, const float* gamma, const float* beta, float eps,
                 const float* bias, int act, int8_t* q, float* s_tok, const DeviceInfo& di,
                 cudaStream_t st) {
    constexpr int EPP = Piece<Tin>::EPP;
    const int idx = pick_shape((int)(H / EPP));
    if (idx < 0 || T > (1ll << 30)) return ZQ_ERR_SHAPE;
    const Shape sh = kShapes[idx];
    const int teams = sh.block / sh.tpr;
    const int row_bytes = (int)(H * sizeof(Tin));
    const int n_par = LN ? 2 : (bias ? 1 : 0);
    const size_t par_bytes = idx < kFirstGlobalParamShape ? (size_t)n_par * H * sizeof(float) : 0;
    // contiguous row ranges, one CTA per SM
    const int64_t grid0 = T < di.sm_count ? T : di.sm_count;
    const int rows_per_cta = (int)((T + grid0 - 1) / grid0);
    const int grid = (int)((T + rows_per_cta - 1) / rows_per_cta);
    // slots per team: as many rows as fit, no more than the team's rows
    int per_team = (int)((kRingBytes - par_bytes) / ((size_t)row_bytes * teams));
    if (per_team > kMaxSlots / teams) per_team = kMaxSlots / teams;
    const int team_rows = (rows_per_cta + teams - 1) / teams;
    if (per_team > team_rows) per_team = team_rows;
    if (per_team < 1) return ZQ_ERR_SHAPE;
    const size_t smem = kRingOffset + par_bytes + (size_t)per_team * teams * row_bytes;
    // exact-fit rows drop the per-piece guards (not for the global-parameter
    // shapes, whose guard-free variants need more registers than they have)
    const bool full = (int64_t)sh.tpr * sh.ppt * EPP == H && idx < kFirstGlobalParamShape;
    auto kern = pipe_kernel<Tin, LN>(idx, full);
    int rc = cuda_status(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    if (rc) return rc;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    cfg.attrs = at;
    cfg.numAttrs = (unsigned)pdl_attr(at[0]);
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3((unsigned)sh.block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    count_launch();
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, x, (int)T, (int)H, 1.0f / (float)H, rows_per_cta, per_team,
                                          gamma, beta, eps, bias, act, q, s_tok, di.status_word));
}

}  // namespace

int launch_rowq_pipe(const void* x, int x_dtype, int64_t T, int64_t H, bool ln, const float* gamma,
                     const float* beta, float eps, const float* bias, int act, int8_t* q,
                     float* s_tok, const DeviceInfo& di, cudaStream_t st) {
    if (x_dtype == ZQ_BF16) {
        const uint16_t* xb = static_cast<const uint16_t*>(x);
        return ln ? launch_typed<uint16_t, true>(xb, T, H, gamma, beta, eps, nullptr, 0, q, s_tok, di, st)
                  : launch_typed<uint16_t, false>(xb, T, H, nullptr, nullptr, 0.f, bias, act, q, s_tok, di, st);
    }
    const float* xf = static_cast<const float*>(x);
    return ln ? launch_typed<float, true>(xf, T, H, gamma, beta, eps, nullptr, 0, q, s_tok, di, st)
              : launch_typed<float, false>(xf, T, H, nullptr, nullptr, 0.f, bias, act, q, s_tok, di, st);
}

}  // namespace zq
