// fa2_bwd.cuh -- FlashAttention-2 backward pass with recomputation for sm_100a.
//
// The handout's backward (CS336 A2 Systems handout section 4.2.2, "backward
// pass with recomputation", Eqs. 13-19):
//   D   = rowsum(O o dO)                       (computed once, before the loop)
//   S   = scale Q K^T,  P_ij = exp(S_ij - L_i)  (Eqs. 13-14, recomputed)
//   dV  = P^T dO,  dP = dO V^T                 (Eqs. 15-16)
//   dS_ij = P_ij (dP_ij - D_i)                 (Eq. 17)
//   dQ  = scale dS K,  dK = scale dS^T Q        (Eqs. 18-19)
// The handout's tiled Algorithm 2 (section 4.2.3) is not printed; it computes
// P twice to avoid atomics.  This file instead uses one pass with the
// key/value tile outermost: dK and dV of a key tile stay in tensor memory for
// the whole pass, and each query tile's dQ contribution is added to an fp32
// accumulator in global memory with vector atomics.
//
// Three kernels, enqueued back to back on one stream:
//   fa2_bwd_pre_kernel   per query row: D_i, L_i * log2(e) (padded to whole
//                        tiles with +inf / 0 so padded rows drop out), and a
//                        zeroed dQ accumulator row.
//   fa2_bwd_kernel       one CTA per (key tile j, head); loops over the query
//                        tiles i that see key tile j (i >= j when causal).
//   fa2_bwd_dq_kernel    dQ = scale * accumulator, rounded to the input type.
#pragma once

#include <cstdint>

#include "fa2_traits.cuh"

namespace fa2 {

// Workspace carved out of the caller's buffer (every region 256-byte aligned).
struct BwdWorkspace {
    size_t l2_off, d_off, dq_off, total;
    int n_pad;
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline BwdWorkspace bwd_workspace_layout(int BH, int N, int d) {
    BwdWorkspace w;
    w.n_pad = (N + kTileRows - 1) / kTileRows * kTileRows;
    const size_t vec = align256(static_cast<size_t>(BH) * w.n_pad * sizeof(float));
    w.l2_off = 0;
    w.d_off = vec;
    w.dq_off = 2 * vec;
    w.total = w.dq_off + align256(static_cast<size_t>(BH) * N * d * sizeof(float));
    return w;
}

// ------------------------------------------------------------------ pre-processing

template <typename T, int D>
__global__ void __launch_bounds__(256)
fa2_bwd_pre_kernel(const T* __restrict__ o, const T* __restrict__ dout,
                   const float* __restrict__ lse, float* __restrict__ l2,
                   float* __restrict__ dvec, float* __restrict__ dq_acc, int N, int n_pad,
                   long long rows_total) {
    const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows_total) return;
    const long long bh = row / n_pad;
    const int n = static_cast<int>(row - bh * n_pad);
    if (n >= N) {
        if (lane == 0) {
            l2[row] = INFINITY;
            dvec[row] = 0.f;
        }
        return;
    }
    const size_t base = (static_cast<size_t>(bh) * N + n) * D;
    float acc = 0.f;
    for (int e = lane; e < D; e += 32) {
        acc += static_cast<float>(o[base + e]) * static_cast<float>(dout[base + e]);
        dq_acc[base + e] = 0.f;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        dvec[row] = acc;
        l2[row] = lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f;
    }
}

// ------------------------------------------------------------------ dQ finalise

template <typename T>
__global__ void __launch_bounds__(256)
fa2_bwd_dq_kernel(const float* __restrict__ dq_acc, T* __restrict__ dq, float scale,
                  long long n4) {
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4 a = reinterpret_cast<const float4*>(dq_acc)[i];
    if constexpr (sizeof(T) == 4) {
        reinterpret_cast<float4*>(dq)[i] = make_float4(a.x * scale, a.y * scale, a.z * scale, a.w * scale);
    } else {
        uint2 w;
        w.x = ptx::pack_bf16x2(a.x * scale, a.y * scale);
        w.y = ptx::pack_bf16x2(a.z * scale, a.w * scale);
        reinterpret_cast<uint2*>(dq)[i] = w;
    }
}

// ------------------------------------------------------------------ main kernel

struct BwdParams {
    const float* l2;       // [BH][n_pad]  L * log2(e), +inf past N
    const float* dvec;     // [BH][n_pad]  D, 0 past N
    float* dq_acc;         // [BH][N][d]   fp32 accumulator (zeroed)
    uint32_t* status;
    int N, BH, n_tiles, n_pad, causal;
    float scale_log2;      // scale * log2(e)
    float scale;
    unsigned long long timeout_ns;
};

template <int ES, int D>
struct BwdCfg {
    using G = TileGeom<ES, D>;
    using GS = TileGeom<ES, 128>;          // a 128 x 128 dS tile, K-major along queries
    using G4 = TileGeom<4, D>;             // the fp32 dQ accumulator's boxes
    static_assert(ES == 2, "the backward kernel is written for 16-bit inputs");
    // One fp32 dQ box (128 rows x kBoxK columns) staged for a TMA reduce-add.
    static constexpr int kStageBytes = kTileRows * G4::kRowBK;
    static constexpr int kThreads = 320;   // 10 warps
    static constexpr int kTile = G::kTileBytesK;
    // 227 KB minus the alignment pad and the static shared memory (per-warp
    // L/D vectors and barriers).
    static constexpr int kBudget = 227 * 1024 - 1024 - 9 * 1024;
    // K, V resident; dS staging; Q_i in a ring of kQSlots, dO_i in a ring of
    // kDOSlots.  Q_i lives from S(i) to dK(i), dO_i from dP(i) to dV(i).
    static constexpr int kFixed = 2 * kTile + GS::kTileBytesK + kStageBytes;
    static constexpr int kSlots0 = (kBudget - kFixed) / kTile;
    static constexpr int kSlots = kSlots0 > 4 ? 4 : kSlots0;
    static_assert(kSlots >= 3, "shared memory too small for the Q/dO rings");
    static constexpr int kQSlots = 2;
    static constexpr int kDOSlots = kSlots - 2;
    static constexpr int kSmemBytes = 1024 + kFixed + kSlots * kTile;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDQ = 128, kColDV = 256, kColDK = 384;
};

// Key/value-tile-outer backward.  One CTA per (key tile j, head), looping over
// the query tiles i that see key tile j.  Per query tile the MMA issuer runs
//   dV += P^T(i) dO(i); S^T(i+1) = K Q(i+1)^T;
//   dK += dS^T(i) Q(i); dQ(i) = dS(i) K; dP^T(i+1) = V dO(i+1)^T
// so that S^T(i+1) overlaps the dS(i) computation and dK(i)/dQ(i)/dP^T(i+1)
// overlap the P(i+1) computation.  Warps: 0 TMA producer, 1 MMA issuer, 2-5
// P/dS warpgroup (one key row per thread), 6-9 dQ warpgroup (one query row per
// thread).
template <int ES, int D>
__global__ void __launch_bounds__(320, 1)
fa2_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
               const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    using Cfg = BwdCfg<ES, D>;
    using G = typename Cfg::G;
    using GS = typename Cfg::GS;
    using G4 = typename Cfg::G4;
    constexpr int QS = Cfg::kQSlots;
    constexpr int DS = Cfg::kDOSlots;
    constexpr int TB = Cfg::kTile;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kv_full;
    __shared__ uint64_t bar_q_full[QS], bar_q_empty[QS], bar_do_full[DS], bar_do_empty[DS];
    __shared__ uint64_t bar_s_full, bar_dp_full, bar_p_ready, bar_ds_ready;
    __shared__ uint64_t bar_dq_full, bar_dq_free, bar_dkv_full, bar_drain;
    __shared__ uint64_t bar_stage_full, bar_stage_free;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    // Per-warp copies of the current query tile's L*log2(e) and D vectors
    // (double-buffered; each warp syncs only itself).
    __shared__ __align__(16) float sL2[4][2][kTileRows];
    __shared__ __align__(16) float sDv[4][2][kTileRows];

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sK = smem;
    uint8_t* sV = sK + TB;
    uint8_t* sDS = sV + TB;
    uint8_t* sQr = sDS + GS::kTileBytesK;
    uint8_t* sDOr = sQr + QS * TB;
    uint8_t* sStage = sDOr + DS * TB;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: with the causal mask, key tile j is seen by query tiles j..T-1,
    // so small j carries the most work and is issued first.
    const int item = blockIdx.x;
    const int kv_tile = item / p.BH;
    const int bh = item - kv_tile * p.BH;
    const int i_begin = p.causal ? kv_tile : 0;
    const int n_q = p.n_tiles - i_begin;
    const int kv_row0 = kv_tile * kTileRows;

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_kv_full, 1);
        for (int s = 0; s < QS; ++s) { ptx::mbar_init(&bar_q_full[s], 1); ptx::mbar_init(&bar_q_empty[s], 1); }
        for (int s = 0; s < DS; ++s) { ptx::mbar_init(&bar_do_full[s], 1); ptx::mbar_init(&bar_do_empty[s], 1); }
        ptx::mbar_init(&bar_s_full, 1);
        ptx::mbar_init(&bar_dp_full, 1);
        ptx::mbar_init(&bar_p_ready, 4);
        ptx::mbar_init(&bar_ds_ready, 4);
        ptx::mbar_init(&bar_dq_full, 1);
        ptx::mbar_init(&bar_dq_free, 4);
        ptx::mbar_init(&bar_dkv_full, 1);
        ptx::mbar_init(&bar_drain, 1);
        ptx::mbar_init(&bar_stage_full, 4);
        ptx::mbar_init(&bar_stage_free, 1);
        ptx::fence_mbar_init();
    }
    if (warp == 1) {
        ptx::tmem_alloc(&tmem_slot, Cfg::kTmemCols);
        ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    const uint64_t tmo = p.timeout_ns;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_do);
            ptx::mbar_arrive_expect_tx(&bar_kv_full, 2 * TB);
            for (int b = 0; b < G::kNBoxK; ++b) {
                ptx::tma_load_3d(sK + b * kTileRows * G::kRowBK, &tm_k, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
                ptx::tma_load_3d(sV + b * kTileRows * G::kRowBK, &tm_v, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
            }
            int q_issued = 0, do_issued = 0;
            for (int it = 0; it < n_q; ++it) {
                const int row0 = (i_begin + it) * kTileRows;
                const int qs = it % QS;
                if (it >= QS && !ptx::mbar_wait(&bar_q_empty[qs], ((it / QS) & 1) ^ 1, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_q_full[qs], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sQr + qs * TB + b * kTileRows * G::kRowBK, &tm_q, &bar_q_full[qs], b * G::kBoxK, row0, bh);
                q_issued = it + 1;
                const int ds = it % DS;
                if (it >= DS && !ptx::mbar_wait(&bar_do_empty[ds], ((it / DS) & 1) ^ 1, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_do_full[ds], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sDOr + ds * TB + b * kTileRows * G::kRowBK, &tm_do, &bar_do_full[ds], b * G::kBoxK, row0, bh);
                do_issued = it + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                ptx::mbar_wait_drain(&bar_kv_full, 0, kDrainNs);
                for (int t = q_issued - 1; t >= 0 && t >= q_issued - QS; --t)
                    ptx::mbar_wait_drain(&bar_q_full[t % QS], (t / QS) & 1, kDrainNs);
                for (int t = do_issued - 1; t >= 0 && t >= do_issued - DS; --t)
                    ptx::mbar_wait_drain(&bar_do_full[t % DS], (t / DS) & 1, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc_s = ptx::instr_desc(G::kFmt, 128, 128, false, false);
            constexpr uint32_t idesc_kv = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            constexpr uint32_t idesc_dq = ptx::instr_desc(G::kFmt, 128, G::kNOut, true, true);
            const uint32_t k_addr = ptx::smem_addr(sK);
            const uint32_t v_addr = ptx::smem_addr(sV);
            const uint32_t ds_addr = ptx::smem_addr(sDS);
            auto q_addr = [&](int it) { return ptx::smem_addr(sQr + (it % QS) * TB); };
            auto do_addr = [&](int it) { return ptx::smem_addr(sDOr + (it % DS) * TB); };
            // S^T = K_j Q_i^T   (Eq. 13, transposed: rows are keys)
            auto issue_s = [&](int it) -> bool {
                if (!ptx::mbar_wait(&bar_q_full[it % QS], (it / QS) & 1, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t qa = q_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColS, desc_kmajor<G>(k_addr, kk), desc_kmajor<G>(qa, kk), idesc_s, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_s_full);
                return true;
            };
            // dP^T = V_j dO_i^T   (Eq. 16, transposed)
            auto issue_dp = [&](int it) -> bool {
                if (!ptx::mbar_wait(&bar_do_full[it % DS], (it / DS) & 1, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t da = do_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColDP, desc_kmajor<G>(v_addr, kk), desc_kmajor<G>(da, kk), idesc_s, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_dp_full);
                return true;
            };
            bool ok = ptx::mbar_wait(&bar_kv_full, 0, &abort_flag, tmo);
            if (ok) ok = issue_s(0) && issue_dp(0);
            for (int it = 0; ok && it < n_q; ++it) {
                // dV_j += P^T dO_i   (Eq. 15), P^T read from the score columns.
                if (!ptx::mbar_wait(&bar_p_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t da = do_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ts(tmem + Cfg::kColDV, tmem + Cfg::kColS + kk * 8, desc_mnmajor<G>(da, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar_do_empty[it % DS]);
                // Next query tile's scores while the P/dS warps work on dS(i).
                if (it + 1 < n_q && !issue_s(it + 1)) { ok = false; break; }
                // dK_j += dS^T Q_i  and  dQ_i = dS K_j   (Eqs. 19 and 18 without the scale)
                if (!ptx::mbar_wait(&bar_ds_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t qa = q_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColDK, desc_kmajor<GS>(ds_addr, kk), desc_mnmajor<G>(qa, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar_q_empty[it % QS]);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColDQ, desc_mnmajor<GS>(ds_addr, kk), desc_mnmajor<G>(k_addr, kk), idesc_dq, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_dq_full);
                // dP^T(i+1) reuses the dQ columns once the dQ warps have read them.
                if (it + 1 < n_q) {
                    if (!ptx::mbar_wait(&bar_dq_free, it & 1, &abort_flag, tmo)) { ok = false; break; }
                    if (!issue_dp(it + 1)) { ok = false; break; }
                }
            }
            if (ok) {
                ptx::mma_commit(&bar_dkv_full);
            } else {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------ P / dS warpgroup
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // key row inside the tile
        const bool key_valid = kv_row0 + r < p.N;
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        const int wq = warp - 2;                          // warp inside the group
        const size_t vec_base = static_cast<size_t>(bh) * p.n_pad;
        float nl2[4], nd[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            nl2[m] = p.l2[vec_base + static_cast<size_t>(i_begin) * kTileRows + lane + 32 * m];
            nd[m] = p.dvec[vec_base + static_cast<size_t>(i_begin) * kTileRows + lane + 32 * m];
        }
        bool ok = true;
        for (int it = 0; it < n_q; ++it) {
            const int i = i_begin + it;
            const int b = it & 1;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                sL2[wq][b][lane + 32 * m] = nl2[m];
                sDv[wq][b][lane + 32 * m] = nd[m];
            }
            __syncwarp();
            if (it + 1 < n_q) {
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    nl2[m] = p.l2[vec_base + static_cast<size_t>(i + 1) * kTileRows + lane + 32 * m];
                    nd[m] = p.dvec[vec_base + static_cast<size_t>(i + 1) * kTileRows + lane + 32 * m];
                }
            }
            const bool diag = p.causal && (i == kv_tile);
            // ---- P^T = exp2(S^T * scale*log2(e) - L*log2(e))   (Eq. 14)
            if (!ptx::mbar_wait(&bar_s_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pk[64];                               // P^T row as bf16 pairs
#pragma unroll
            for (int h0 = 0; h0 < 128; h0 += 32) {
                uint32_t us[32];
                ptx::tmem_ld32(lane_base + Cfg::kColS + h0, us);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 lv = *reinterpret_cast<const float4*>(&sL2[wq][b][h0 + c]);
                    const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
                    float pv[4];
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        const int q = h0 + c + h;
                        float pe = ptx::ex2_approx(fmaf(__uint_as_float(us[c + h]), sl2, -lq[h]));
                        if ((diag && r > q) || !key_valid) pe = 0.f;
                        pv[h] = pe;
                    }
                    pk[(h0 + c) >> 1] = ptx::pack_bf16x2(pv[0], pv[1]);
                    pk[((h0 + c) >> 1) + 1] = ptx::pack_bf16x2(pv[2], pv[3]);
                }
            }
            // P^T -> TMEM score columns [0, 64) as the A operand of dV += P^T dO.
            ptx::tmem_st32(lane_base + Cfg::kColS, *reinterpret_cast<uint32_t(*)[32]>(pk));
            ptx::tmem_st32(lane_base + Cfg::kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(pk + 32));
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_p_ready);
            // ---- dS^T = P^T o (dP^T - D)   (Eq. 17) -> shared memory
            if (!ptx::mbar_wait(&bar_dp_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t ud[32];
                ptx::tmem_ld32(lane_base + Cfg::kColDP + c0, ud);
                ptx::tmem_wait_ld();
                uint32_t dw[16];
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 dv4 = *reinterpret_cast<const float4*>(&sDv[wq][b][c0 + c]);
                    const float dq4[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
                    for (int h = 0; h < 4; h += 2) {
                        const uint32_t pw = pk[(c0 + c + h) >> 1];
                        const float p0 = __uint_as_float(pw << 16);
                        const float p1 = __uint_as_float(pw & 0xffff0000u);
                        const float d0 = p0 * (__uint_as_float(ud[c + h]) - dq4[h]);
                        const float d1 = p1 * (__uint_as_float(ud[c + h + 1]) - dq4[h + 1]);
                        dw[(c + h) >> 1] = ptx::pack_bf16x2(d0, d1);
                    }
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    uint4 w = make_uint4(dw[4 * k4], dw[4 * k4 + 1], dw[4 * k4 + 2], dw[4 * k4 + 3]);
                    *reinterpret_cast<uint4*>(sDS + kmajor_chunk_offset<GS>(r, c0 + 8 * k4)) = w;
                }
            }
            ptx::fence_async_smem();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_ds_ready);
        }
        // ---------------- epilogue: dK, dV rows -> shared memory -> TMA store.
        if (ok) ok = ptx::mbar_wait(&bar_dkv_full, 0, &abort_flag, tmo);
        if (ok) {
            ptx::tc_fence_after();
#pragma unroll
            for (int which = 0; which < 2; ++which) {
                const uint32_t col = which == 0 ? Cfg::kColDV : Cfg::kColDK;
                const float mul = which == 0 ? 1.f : p.scale;
                uint8_t* stage = which == 0 ? sV : sK;
#pragma unroll
                for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                    uint32_t u[16];
                    ptx::tmem_ld16(lane_base + col + c0, u);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int cc = c0 + 8 * h8;
                        if (cc < D) {
                            const float* f = reinterpret_cast<const float*>(u) + 8 * h8;
                            uint4 w;
                            w.x = ptx::pack_bf16x2(f[0] * mul, f[1] * mul);
                            w.y = ptx::pack_bf16x2(f[2] * mul, f[3] * mul);
                            w.z = ptx::pack_bf16x2(f[4] * mul, f[5] * mul);
                            w.w = ptx::pack_bf16x2(f[6] * mul, f[7] * mul);
                            *reinterpret_cast<uint4*>(stage + kmajor_chunk_offset<G>(r, cc)) = w;
                        }
                    }
                }
            }
            ptx::fence_async_smem();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok && threadIdx.x == 64) {
            for (int b = 0; b < G::kNBoxK; ++b) {
                ptx::tma_store_3d(&tm_dv, sV + b * kTileRows * G::kRowBK, b * G::kBoxK, kv_row0, bh);
                ptx::tma_store_3d(&tm_dk, sK + b * kTileRows * G::kRowBK, b * G::kBoxK, kv_row0, bh);
            }
            ptx::tma_store_commit();
            ptx::tma_store_wait_all();
        }
    } else {
        // ------------------------------------------------ dQ warpgroup
        // Drains each dQ tile from TMEM into registers (so the next dP^T MMA
        // can reuse the columns), then adds it into the fp32 accumulator one
        // box of columns at a time: rows are written to a swizzled staging box
        // in shared memory and one thread issues a TMA reduce-add, which does
        // the additions in L2 without occupying the SM's load/store path.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // query row inside tile i
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const bool issuer = threadIdx.x == 192;
        constexpr int NB4 = G4::kNBoxK;
        constexpr int kChunks = G4::kRowBK / 16;         // 16-byte chunks per staged row
        bool ok = true;
        for (int it = 0; it < n_q && ok; ++it) {
            const int q_row0 = (i_begin + it) * kTileRows;
            if (!ptx::mbar_wait(&bar_dq_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t u[G::kNOut];
#pragma unroll
            for (int c0 = 0; c0 < G::kNOut; c0 += 16)
                ptx::tmem_ld16(lane_base + Cfg::kColDQ + c0, *reinterpret_cast<uint32_t(*)[16]>(u + c0));
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_dq_free);
#pragma unroll
            for (int c = 0; c < NB4; ++c) {
                const int round = it * NB4 + c;
                if (round > 0 && !ptx::mbar_wait(&bar_stage_free, (round - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
#pragma unroll
                for (int k = 0; k < kChunks; ++k) {
                    const int col = c * G4::kBoxK + 4 * k;
                    if (col < D) {
                        const int sw = ((r * G4::kRowBK) >> 7) & (kChunks - 1);
                        *reinterpret_cast<uint4*>(sStage + r * G4::kRowBK + ((k ^ sw) * 16)) =
                            make_uint4(u[col], u[col + 1], u[col + 2], u[col + 3]);
                    }
                }
                ptx::fence_async_smem();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_stage_full);
                if (issuer) {
                    if (!ptx::mbar_wait(&bar_stage_full, round & 1, &abort_flag, tmo)) { ok = false; break; }
                    ptx::tma_reduce_add_3d(&tm_dq, sStage, c * G4::kBoxK, q_row0, bh);
                    ptx::tma_store_commit();
                    ptx::tma_store_wait_read_all();
                    ptx::mbar_arrive(&bar_stage_free);
                }
            }
        }
        if (issuer) ptx::tma_store_wait_all();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    if (threadIdx.x == 0 && abort_flag) atomicCAS(p.status, 0u, kDevStatusTimeout);
}

}  // namespace fa2
