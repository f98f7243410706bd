// fa2_bwd_fused.cuh -- one-pass FlashAttention-2 backward for sm_100a: a
// key-tile-outer loop that produces dK, dV and the dQ contributions together.
//
// The same equations as fa2_bwd.cuh (CS336 A2 Systems handout section 4.2.2,
// Eqs. 13-19, D = rowsum(O o dO)), organised with the key/value tile outermost
// as in the FlashAttention-2 backward the handout describes before Algorithm 2:
// P is computed once per (key tile, query tile) pair, and the contribution
//   dQ_i += scale dS_ij K_j                                   (Eq. 18)
// of key tile j to query tile i is added into an fp32 accumulator dQ_acc in
// global memory with TMA reduce-add.  Five tensor-core products per tile pair
// instead of the seven of the two-pass form (which recomputes S and dP for dQ),
// at the price of dQ bits that depend on the order in which the key tiles'
// contributions arrive (dK and dV stay deterministic).
//
// One CTA per (key tile j, key/value head), 16 warps:
//   warp 0       TMA producer: K_j, V_j once; Q_i, dO_i through two rings.
//   warp 1       MMA issuer (one thread), per query tile i:
//                  S^T  = K_j Q_i^T            (SS)      -> TMEM
//                  dP^T = V_j dO_i^T           (SS)      -> TMEM
//                  dV  += P^T dO_i             (TS, P^T from TMEM)
//                  dK  += dS^T Q_i             (SS, dS^T from shared memory)
//                  dQ_i = dS K_j               (SS, dS read M-major from the
//                                               same shared-memory tile) -> TMEM
//   warps 4-11   two elementwise groups (query columns [64g, 64g + 64) of the
//                tile): P^T = exp2(S^T scale log2(e) - L log2(e)) back into
//                TMEM as 16-bit pairs; dS^T = P^T o (dP^T - D) as 16-bit
//                values into the shared-memory dS tile.
//   warps 12-15  dQ drain: read dQ_i from TMEM in 32-column chunks, stage them
//                in the dS tile (free once dK and dQ have read it) and add
//                them to dQ_acc with cp.reduce.async.bulk.tensor.
// Warp 2 and 3 idle.  A finalisation kernel scales dQ_acc and rounds it to
// the input type.
//
// Query tiles whose rows see only this key tile (causal: the first query tile;
// or a single key tile) are not accumulated here: their dQ, and their D in the
// form sum_j P_ij dP_ij, come from the query-tile pass of fa2_bwd.cuh run on
// those tiles beforehand (see fa2_bwd.cuh); for them this kernel passes dS^T
// to the dK product as hi (shared memory) + lo (TMEM) 16-bit parts.
//
// Tensor memory (512 columns): S^T | dP^T | dV | dK, with dQ_i in the dP^T
// columns when the head dimension leaves no room (d = 80, 128; the issuer then
// waits for the drain before the next dP^T), else in its own columns.
#pragma once

#include <cstdint>

#include "fa2_bwd.cuh"
#include "fa2_traits.cuh"

namespace fa2 {

template <int ES, int D, bool F16 = false>
struct BwdFusedCfg {
    using G = TileGeom<ES, D, F16>;
    using GS = TileGeom<2, 128, F16>;     // the dS tile: 128 key rows x 128 query columns
    static_assert(ES == 2, "the one-pass backward is written for 16-bit inputs");
    static constexpr int kThreads = 512;
    static constexpr int kTile = G::kTileBytesK;
    static constexpr int kDsBytes = GS::kTileBytesK;          // 32 KB
    // 227 KB minus the alignment pad and the (small) static shared memory.
    static constexpr int kBudget = 227 * 1024 - 1024 - 1024;
    static constexpr int kRing0 = (kBudget - 2 * kTile - kDsBytes) / (2 * kTile);
    static constexpr int kRing = kRing0 > 3 ? 3 : kRing0;
    static_assert(kRing >= 2, "shared memory too small for the streaming rings");
    static constexpr int kSmemBase = 1024 + 2 * kTile + 2 * kRing * kTile + kDsBytes;
    // Tensor memory.
    static constexpr uint32_t kTmemCols = 512;
    // d > 64 (d = 80, 128): S^T | dP^T (and dQ_i) | dV | dK at columns 0, 128,
    // 256, 384.  d <= 64: S^T | dP^T | dV | dK | dQ_i, each accumulator d wide.
    static constexpr uint32_t kColS = 0, kColDP = 128;
    static constexpr bool kDqInDp = G::kNOut > 64;
    static constexpr uint32_t kColDV = 256;
    static constexpr uint32_t kColDK = kDqInDp ? 384 : 256 + G::kNOut;
    static constexpr uint32_t kColDQ = kDqInDp ? kColDP : 256 + 2 * G::kNOut;
    static_assert(kColDK + G::kNOut <= 512 && kColDQ + G::kNOut <= 512, "tensor memory overflow");
    // dQ drain: chunks of kCW fp32 columns, staged in halves of the dS tile (free
    // once dK and dQ have read it).
    static constexpr int kCW = G::kNOut >= 32 ? 32 : G::kNOut;
    static constexpr int kNCh = (G::kNOut + kCW - 1) / kCW;
    static constexpr int kChunkBytes = kTileRows * kCW * 4;
    static_assert(2 * kChunkBytes <= kDsBytes, "two drain chunks must fit in the dS tile");
    // Where shared memory allows (d <= 64), dQ_i is staged in a buffer of its own
    // that outlives the step, so the dS tile is free as soon as dK and dQ have
    // read it; at d = 80 and 128 the staging shares the dS tile.
    static constexpr bool kOwnStage = kSmemBase + kNCh * kChunkBytes <= kBudget + 1024;
    static constexpr int kSmemBytes = kSmemBase + (kOwnStage ? kNCh * kChunkBytes : 0);
    // Register split (512 threads launch with 128 registers each): warpgroup 0
    // (producer, issuer) and the drain warpgroup give registers to the two
    // elementwise warpgroups.
    static constexpr int kLaunchRegs = 128;
    static constexpr int kRegsLow = 88;
    static constexpr int kRegsEw = 152;
    static constexpr int kRegsDrain = 120;
    static_assert(128 * kRegsLow + 256 * kRegsEw + 128 * kRegsDrain <= kThreads * kLaunchRegs,
                  "register split exceeds the registers the block is launched with");
};

// Staging offset of 16-byte unit u (4 fp32 values) of row r in a chunk of kCW
// fp32 columns, in the layout the TMA's 128-byte (kCW = 32) or 64-byte
// (kCW = 16) swizzle expects (which also spreads a warp's row writes over all
// banks).
template <int kCW>
__device__ __forceinline__ uint32_t stage_offset(int r, int u) {
    if constexpr (kCW == 32) return r * 128 + ((u ^ (r & 7)) << 4);
    else return r * 64 + ((u ^ ((r >> 1) & 3)) << 4);
}

// A query tile whose rows see no key tile but one: its D (in the form
// sum_j P_ij dP_ij) and its dQ come from the query-tile pass beforehand.
__device__ __forceinline__ bool fused_single_tile(const BwdParams& p, int q_tile) {
    return p.n_tiles_k == 1 || (p.causal && q_tile == 0);
}

template <int ES, int D, bool F16 = false>
__global__ void __launch_bounds__(512, 1)
fa2_bwd_fused_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                     const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = BwdFusedCfg<ES, D, F16>;
    using G = typename Cfg::G;
    using GS = typename Cfg::GS;
    constexpr int RS = Cfg::kRing;
    constexpr int TB = Cfg::kTile;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kv_full;
    __shared__ uint64_t bar_q_full[RS], bar_q_empty[RS], bar_do_full[RS], bar_do_empty[RS];
    __shared__ uint64_t bar_s_full, bar_dp_full, bar_p_ready, bar_ds_ready;
    __shared__ uint64_t bar_dq_full, bar_dq_drained, bar_ds_free;
    __shared__ uint64_t bar_dkv_full, bar_drain;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    __shared__ volatile uint32_t drain_ok;

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sK = smem;
    uint8_t* sV = sK + TB;
    uint8_t* sQr = sV + TB;
    uint8_t* sDOr = sQr + RS * TB;
    uint8_t* sDS = sDOr + RS * TB;
    uint8_t* sStage = Cfg::kOwnStage ? sDS + Cfg::kDsBytes : sDS;    // dQ staging

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: (key tile j, key/value head), in groups of p.head_group heads
    // (grouped_item: the CTAs resident together share those heads' Q, dO and dQ
    // accumulator in L2); inside a group key tile 0, which the most query tiles
    // see under the causal rule, comes first.
    int kv_tile, bh;                                     // bh: key/value head
    grouped_item(blockIdx.x, p.n_tiles_k, p.BH_kv, p.head_group, kv_tile, bh);
    const int i_begin = p.causal ? kv_tile : 0;
    const int kv_row0 = kv_tile * kTileRows;
    const int n_q = p.n_tiles > i_begin ? p.n_tiles - i_begin : 0;
    const int n_it = n_q * p.group;                      // (query head, query tile) steps
    auto q_tile_of = [&](int it) { return i_begin + it % n_q; };
    auto q_head_of = [&](int it) { return (bh / p.H_kv) * p.H + (bh % p.H_kv) * p.group + it / n_q; };
    auto single_of = [&](int it) { return fused_single_tile(p, q_tile_of(it)); };

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_kv_full, 1);
        for (int s = 0; s < RS; ++s) {
            ptx::mbar_init(&bar_q_full[s], 1);
            ptx::mbar_init(&bar_q_empty[s], 1);
            ptx::mbar_init(&bar_do_full[s], 1);
            ptx::mbar_init(&bar_do_empty[s], 1);
        }
        ptx::mbar_init(&bar_s_full, 1);
        ptx::mbar_init(&bar_dp_full, 1);
        ptx::mbar_init(&bar_p_ready, 8);
        ptx::mbar_init(&bar_ds_ready, 8);
        ptx::mbar_init(&bar_dq_full, 1);
        ptx::mbar_init(&bar_dq_drained, 4);
        ptx::mbar_init(&bar_ds_free, 1);
        ptx::mbar_init(&bar_dkv_full, 1);
        ptx::mbar_init(&bar_drain, 1);
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

    if (warp < 4) {
    ptx::setmaxnreg_dec<Cfg::kRegsLow>();
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_it > 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_do);
            ptx::mbar_arrive_expect_tx(&bar_kv_full, 2 * TB);
            for (int b = 0; b < G::kNBoxK; ++b) {
                ptx::tma_load_3d(sK + b * kTileRows * G::kRowBK, &tm_k, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
                ptx::tma_load_3d(sV + b * kTileRows * G::kRowBK, &tm_v, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
            }
            int q_issued = 0, do_issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int row0 = q_tile_of(it) * kTileRows;
                const int qh = q_head_of(it);
                const int s = it % RS;
                const uint32_t ph = ((it / RS) & 1) ^ 1;
                if (it >= RS && !ptx::mbar_wait(&bar_q_empty[s], ph, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_q_full[s], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sQr + s * TB + b * kTileRows * G::kRowBK, &tm_q, &bar_q_full[s], b * G::kBoxK, row0, qh);
                q_issued = it + 1;
                if (it >= RS && !ptx::mbar_wait(&bar_do_empty[s], ph, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_do_full[s], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sDOr + s * TB + b * kTileRows * G::kRowBK, &tm_do, &bar_do_full[s], b * G::kBoxK, row0, qh);
                do_issued = it + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                ptx::mbar_wait_drain(&bar_kv_full, 0, kDrainNs);
                for (int t = q_issued - 1; t >= 0 && t >= q_issued - RS; --t)
                    ptx::mbar_wait_drain(&bar_q_full[t % RS], (t / RS) & 1, kDrainNs);
                for (int t = do_issued - 1; t >= 0 && t >= do_issued - RS; --t)
                    ptx::mbar_wait_drain(&bar_do_full[t % RS], (t / RS) & 1, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n_it > 0) {
            constexpr uint32_t idesc_s = ptx::instr_desc(G::kFmt, 128, 128, false, false);
            constexpr uint32_t idesc_kv = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            constexpr uint32_t idesc_dq = ptx::instr_desc(G::kFmt, 128, G::kNOut, true, true);
            const uint32_t k_addr = ptx::smem_addr(sK);
            const uint32_t v_addr = ptx::smem_addr(sV);
            const uint32_t ds_addr = ptx::smem_addr(sDS);
            auto q_addr = [&](int it) { return ptx::smem_addr(sQr + (it % RS) * TB); };
            auto do_addr = [&](int it) { return ptx::smem_addr(sDOr + (it % RS) * TB); };
            // S^T = K_j Q_i^T (Eq. 13, transposed).  Q_i / dO_i of step i >= 1 have
            // landed once the groups report P^T / dS^T of step i-1 (one thread
            // checks them before arriving), so only step 0 waits on the loads here.
            auto issue_s = [&](int it) -> bool {
                if (it == 0 && !ptx::mbar_wait(&bar_q_full[0], 0, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t qa = q_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColS, desc_kmajor<G>(k_addr, kk), desc_kmajor<G>(qa, kk), idesc_s, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_s_full);
                return true;
            };
            // dP^T = V_j dO_i^T (Eq. 16, transposed)
            auto issue_dp = [&](int it) -> bool {
                if (it == 0 && !ptx::mbar_wait(&bar_do_full[0], 0, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t da = do_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColDP, desc_kmajor<G>(v_addr, kk), desc_kmajor<G>(da, kk), idesc_s, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_dp_full);
                return true;
            };
            int n_dq = 0;                                 // dQ products issued so far
            bool ok = ptx::mbar_wait(&bar_kv_full, 0, &abort_flag, tmo);
            if (ok) ok = issue_s(0) && issue_dp(0);
            for (int it = 0; ok && it < n_it; ++it) {
                const bool single = single_of(it);
                // dV_j += P^T dO_i   (Eq. 15); P^T read from the score columns.
                if (!ptx::mbar_wait(&bar_p_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t da = do_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ts(tmem + Cfg::kColDV, tmem + Cfg::kColS + a_col(kk), desc_mnmajor<G>(da, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar_do_empty[it % RS]);
                if (it + 1 < n_it && !issue_s(it + 1)) { ok = false; break; }
                // dK_j += dS^T Q_i   (Eq. 19 without the scale); dS^T from shared memory.
                if (!ptx::mbar_wait(&bar_ds_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t qa = q_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ss(tmem + Cfg::kColDK, desc_kmajor<GS>(ds_addr, kk), desc_mnmajor<G>(qa, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                if (single) {
                    // dK_j += dS^T_lo Q_i: the low parts in the dP^T columns.
#pragma unroll
                    for (int kk = 0; kk < G::kStepsRows; ++kk)
                        ptx::mma_f16_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDP + a_col(kk), desc_mnmajor<G>(qa, kk), idesc_kv, 1u);
                    ptx::mma_commit(&bar_q_empty[it % RS]);
                    ptx::mma_commit(&bar_ds_free);           // dS tile read: free for the next step
                } else {
                    ptx::mma_commit(&bar_q_empty[it % RS]);
                    // dQ_i = dS K_j   (Eq. 18 without the scale): A = dS read M-major
                    // from the dS^T tile, B = K_j read N-major.  With separate dQ
                    // columns the previous drain must have read them first.
                    if (!Cfg::kDqInDp && n_dq > 0 &&
                        !ptx::mbar_wait(&bar_dq_drained, (n_dq - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
#pragma unroll
                    for (int kk = 0; kk < G::kStepsRows; ++kk)
                        ptx::mma_f16_ss(tmem + Cfg::kColDQ, desc_mnmajor<GS>(ds_addr, kk), desc_mnmajor<G>(k_addr, kk), idesc_dq, kk > 0 ? 1u : 0u);
                    ptx::mma_commit(&bar_dq_full);
                    // With its own staging the drain leaves the dS tile alone.
                    if (Cfg::kOwnStage) ptx::mma_commit(&bar_ds_free);
                    ++n_dq;
                    // dQ shares the dP^T columns: the next dP^T waits for the drain.
                    if (Cfg::kDqInDp && it + 1 < n_it &&
                        !ptx::mbar_wait(&bar_dq_drained, (n_dq - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
                }
                if (it + 1 < n_it && !issue_dp(it + 1)) { ok = false; break; }
            }
            if (ok) {
                ptx::mma_commit(&bar_dkv_full);
            } else {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    }
    } else if (warp < 12) {
        ptx::setmaxnreg_inc<Cfg::kRegsEw>();
        // ------------------------------------------------ two P / dS groups
        const int g = (warp - 4) >> 2;                  // query columns [64g, 64g+64)
        const int wi = warp - 4;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // key row inside the tile
        const int qc0 = 64 * g;
        const bool key_valid = kv_row0 + r < p.Nk;
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = q_tile_of(it);
            const bool diag = p.causal && (i == kv_tile);
            const bool single = single_of(it);
            // This group's 64 query columns of the L*log2(e) and D vectors.
            const size_t vb = static_cast<size_t>(q_head_of(it)) * p.n_pad + static_cast<size_t>(i) * kTileRows + qc0;
            const float4* l2v = reinterpret_cast<const float4*>(p.l2 + vb);
            const float4* dv4 = reinterpret_cast<const float4*>(p.dvec + vb);
            if (it + 1 < n_it && lane < 8) {
                // Bring the next step's L*log2(e) and D (512 bytes each) into L1 early.
                const size_t nb = static_cast<size_t>(q_head_of(it + 1)) * p.n_pad +
                                  static_cast<size_t>(q_tile_of(it + 1)) * kTileRows + 32 * (lane & 3);
                const float* src = (lane < 4 ? p.l2 : p.dvec) + nb;
                asm volatile("prefetch.global.L1 [%0];" ::"l"(src));
            }
            // ---- P^T = exp2(S^T * scale*log2(e) - L*log2(e))   (Eq. 14)
            if (!ptx::mbar_wait(&bar_s_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pk[32];                               // this group's P^T row, 16-bit pairs
            {
                uint32_t us[64];
                ptx::tmem_ld32(lane_base + Cfg::kColS + qc0, *reinterpret_cast<uint32_t(*)[32]>(us));
                ptx::tmem_ld32(lane_base + Cfg::kColS + qc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(us + 32));
                ptx::tmem_wait_ld();
                const float2 sl2v = make_float2(sl2, sl2);
                if (diag || !key_valid) {
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 lv = __ldg(l2v + (c >> 2));
                        const float2 a0 = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, make_float2(-lv.x, -lv.y));
                        const float2 a1 = ptx::fma2(make_float2(__uint_as_float(us[c + 2]), __uint_as_float(us[c + 3])), sl2v, make_float2(-lv.z, -lv.w));
                        float pv[4] = {ptx::ex2_approx(a0.x), ptx::ex2_approx(a0.y), ptx::ex2_approx(a1.x), ptx::ex2_approx(a1.y)};
#pragma unroll
                        for (int h = 0; h < 4; ++h)
                            if ((diag && r > qc0 + c + h) || !key_valid) pv[h] = 0.f;
                        pk[c >> 1] = G::pack2(pv[0], pv[1]);
                        pk[(c >> 1) + 1] = G::pack2(pv[2], pv[3]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 lv = __ldg(l2v + (c >> 2));
                        const float2 a0 = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, make_float2(-lv.x, -lv.y));
                        const float2 a1 = ptx::fma2(make_float2(__uint_as_float(us[c + 2]), __uint_as_float(us[c + 3])), sl2v, make_float2(-lv.z, -lv.w));
                        pk[c >> 1] = G::pack2(ptx::ex2_approx(a0.x), ptx::ex2_approx(a0.y));
                        pk[(c >> 1) + 1] = G::pack2(ptx::ex2_approx(a1.x), ptx::ex2_approx(a1.y));
                    }
                }
            }
            // P^T -> this group's own score columns [64g, 64g + 32), A operand of
            // dV += P^T dO.
            ptx::tmem_st32(lane_base + Cfg::kColS + qc0, pk);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                // The issuer's S^T(it+1) follows this barrier: check Q_{it+1} first.
                if (wi == 0 && it + 1 < n_it)
                    ok = ptx::mbar_wait(&bar_q_full[(it + 1) % RS], ((it + 1) / RS) & 1, &abort_flag, tmo);
                if (ok) ptx::mbar_arrive(&bar_p_ready);
            }
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
            // ---- dS^T = P^T o (dP^T - D)   (Eq. 17)
            if (!ptx::mbar_wait(&bar_dp_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            // dS^T (16-bit) for this group's 64 query columns, in two halves of 32; on
            // single-tile steps also the rounding remainders (lo parts), which go to
            // this group's dP^T columns (already read), the A operand of the issuer's
            // second dK product.
            uint32_t dk[32];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t ud[32], dl[16];
                ptx::tmem_ld32(lane_base + Cfg::kColDP + qc0 + 32 * h, ud);
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 d4 = __ldg(dv4 + ((32 * h + c) >> 2));
                    const float2 nd[2] = {make_float2(-d4.x, -d4.y), make_float2(-d4.z, -d4.w)};
#pragma unroll
                    for (int e = 0; e < 4; e += 2) {
                        float2 pp;
                        G::unpack2(pk[(32 * h + c + e) >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c + e]), __uint_as_float(ud[c + e + 1])), nd[e >> 1]));
                        const int wd = (32 * h + c + e) >> 1;
                        dk[wd] = G::pack2(ds.x, ds.y);
                        if (single) {
                            float2 hv;
                            G::unpack2(dk[wd], hv.x, hv.y);
                            dl[(c + e) >> 1] = G::pack2(ds.x - hv.x, ds.y - hv.y);
                        }
                    }
                }
                if (single) ptx::tmem_st16(lane_base + Cfg::kColDP + qc0 + 16 * h, dl);
            }
            // -> the shared-memory dS tile (row r, query columns [64g, 64g + 64)), once
            // the previous step's products and dQ drain have released it.
            if (it > 0 && !ptx::mbar_wait(&bar_ds_free, (it - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
#pragma unroll
            for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(sDS + kmajor_chunk_offset<GS>(r, qc0 + 8 * u)) =
                    make_uint4(dk[4 * u], dk[4 * u + 1], dk[4 * u + 2], dk[4 * u + 3]);
            ptx::fence_async_smem();
            if (single) ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                // The issuer's dP^T(it+1) follows this barrier: check dO_{it+1} first.
                if (wi == 0 && it + 1 < n_it)
                    ok = ptx::mbar_wait(&bar_do_full[(it + 1) % RS], ((it + 1) / RS) & 1, &abort_flag, tmo);
                if (ok) ptx::mbar_arrive(&bar_ds_ready);
            }
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) { ok = false; break; }
        }
        // ---------------- epilogue: dV (group 0) / dK (group 1) -> shared memory -> TMA store
        // (zeros when no query reaches this key tile).
        if (ok && n_it > 0) ok = ptx::mbar_wait(&bar_dkv_full, 0, &abort_flag, tmo);
        uint8_t* out_stage = g == 0 ? sV : sK;
        if (ok) {
            ptx::tc_fence_after();
            const uint32_t col = g == 0 ? Cfg::kColDV : Cfg::kColDK;
            const float mul = g == 0 ? 1.f : p.scale;
#pragma unroll
            for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                uint32_t u[16] = {};
                if (n_it > 0) {
                    ptx::tmem_ld16(lane_base + col + c0, u);
                    ptx::tmem_wait_ld();
                }
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int cc = c0 + 8 * h8;
                    if (cc < D) {
                        const float* f = reinterpret_cast<const float*>(u) + 8 * h8;
                        uint4 w;
                        w.x = G::pack2(f[0] * mul, f[1] * mul);
                        w.y = G::pack2(f[2] * mul, f[3] * mul);
                        w.z = G::pack2(f[4] * mul, f[5] * mul);
                        w.w = G::pack2(f[6] * mul, f[7] * mul);
                        *reinterpret_cast<uint4*>(out_stage + kmajor_chunk_offset<G>(r, cc)) = w;
                    }
                }
            }
            ptx::fence_async_smem();
        }
        if (g == 0)
            asm volatile("bar.sync 1, 128;" ::: "memory");
        else
            asm volatile("bar.sync 2, 128;" ::: "memory");
        if (ok && (threadIdx.x & 127) == 64) {
            const CUtensorMap* out_map = g == 0 ? &tm_dv : &tm_dk;
            for (int bx = 0; bx < G::kNBoxK; ++bx)
                ptx::tma_store_3d(out_map, out_stage + bx * kTileRows * G::kRowBK, bx * G::kBoxK, kv_row0, bh);
            ptx::tma_store_commit();
            ptx::tma_store_wait_all();
        }
    } else {
        ptx::setmaxnreg_dec<Cfg::kRegsDrain>();
        // ------------------------------------------------ dQ drain (warps 12-15)
        // Thread t owns query row t of the tile (TMEM lane t).  Per step with a
        // dQ product, dQ_i leaves TMEM in kCW-column chunks of one row per thread:
        // the first two chunks into the two halves of the dS tile (free once dK
        // and dQ have read it), in the layout of the TMA's swizzle, the others
        // into registers, so that TMEM is released after the loads alone.  One
        // thread then adds the staged chunks to dQ_acc with TMA reduce-add
        // (cp.reduce.async.bulk.tensor), waits until the copies have read them,
        // and the register chunks follow through the same halves.  The copy
        // engine performs the additions in L2, away from the SM's load/store
        // queues, which the other roles keep using.  The dS tile is released
        // once the last copy has read it.  That thread takes every wait; the
        // others follow it through a named barrier.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const bool leader = threadIdx.x == 384;
        constexpr int kU = Cfg::kCW / 4;                   // 16-byte units per chunk row
        constexpr int kInSmem = Cfg::kOwnStage ? Cfg::kNCh : (Cfg::kNCh < 2 ? Cfg::kNCh : 2);
        constexpr int kInRegs = Cfg::kNCh - kInSmem;       // 0, 1 (d = 80) or 2 (d = 128)
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        auto load_chunk = [&](int c, uint32_t (&u)[Cfg::kCW]) {
            if constexpr (Cfg::kCW == 32)
                ptx::tmem_ld32(lane_base + Cfg::kColDQ + c * Cfg::kCW, *reinterpret_cast<uint32_t(*)[32]>(u));
            else
                ptx::tmem_ld16(lane_base + Cfg::kColDQ + c * Cfg::kCW, *reinterpret_cast<uint32_t(*)[16]>(u));
            ptx::tmem_wait_ld();
        };
        auto put_row = [&](uint8_t* st, const uint32_t (&u)[Cfg::kCW]) {   // this thread's row
#pragma unroll
            for (int q4 = 0; q4 < kU; ++q4)
                *reinterpret_cast<uint4*>(st + stage_offset<Cfg::kCW>(r, q4)) =
                    make_uint4(u[4 * q4], u[4 * q4 + 1], u[4 * q4 + 2], u[4 * q4 + 3]);
        };
        int n_dq = 0;
        for (int it = 0; it < n_it; ++it) {
            if (single_of(it)) continue;
            if (leader) drain_ok = ptx::mbar_wait(&bar_dq_full, n_dq & 1, &abort_flag, tmo) ? 1u : 0u;
            asm volatile("bar.sync 4, 128;" ::: "memory");
            if (!drain_ok) break;
            ptx::tc_fence_after();
            const int q_row0 = q_tile_of(it) * kTileRows;
            const int qh = q_head_of(it);
            uint32_t keep[kInRegs > 0 ? kInRegs : 1][Cfg::kCW];
            if (Cfg::kOwnStage) {
                // The previous step's copies must have read the staging buffer.
                if (leader) ptx::tma_store_wait_read_all();
                asm volatile("bar.sync 4, 128;" ::: "memory");
            }
#pragma unroll
            for (int c = 0; c < kInSmem; ++c) {
                uint32_t u[Cfg::kCW];
                load_chunk(c, u);
                put_row(sStage + c * Cfg::kChunkBytes, u);
            }
#pragma unroll
            for (int c = 0; c < kInRegs; ++c) load_chunk(kInSmem + c, keep[c]);
            // Every column of dQ_i has left TMEM: the issuer may reuse them.
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_dq_drained);
            ptx::fence_async_smem();
            asm volatile("bar.sync 4, 128;" ::: "memory");
            if (leader) {
#pragma unroll
                for (int c = 0; c < kInSmem; ++c)
                    ptx::tma_reduce_add_3d(&tm_dqacc, sStage + c * Cfg::kChunkBytes, c * Cfg::kCW, q_row0, qh);
                ptx::tma_store_commit();
                if (kInRegs > 0) ptx::tma_store_wait_read_all();
            }
            if (kInRegs > 0) {
                asm volatile("bar.sync 4, 128;" ::: "memory");    // the halves have been read
#pragma unroll
                for (int c = 0; c < kInRegs; ++c) put_row(sDS + c * Cfg::kChunkBytes, keep[c]);
                ptx::fence_async_smem();
                asm volatile("bar.sync 4, 128;" ::: "memory");
                if (leader) {
#pragma unroll
                    for (int c = 0; c < kInRegs; ++c)
                        ptx::tma_reduce_add_3d(&tm_dqacc, sDS + c * Cfg::kChunkBytes, (kInSmem + c) * Cfg::kCW, q_row0, qh);
                    ptx::tma_store_commit();
                }
            }
            if (leader && !Cfg::kOwnStage) {
                // The copies have read the dS tile: the groups may refill it.
                ptx::tma_store_wait_read_all();
                ptx::mbar_arrive(&bar_ds_free);
            }
            ++n_dq;
        }
        if (leader) ptx::tma_store_wait_all();
    }

    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        ptx::tc_fence_after();
        ptx::tmem_dealloc(tmem, Cfg::kTmemCols);
    }
    if (threadIdx.x == 0 && abort_flag) atomicCAS(p.status, 0u, kDevStatusTimeout);
}

// dQ = scale * dQ_acc rounded once to the 16-bit type, for the query rows the
// one-pass kernel accumulated (rows of single-tile query tiles were written by
// the query-tile pass and are left alone).  One thread per 8 consecutive
// columns of a row.
template <bool F16>
__global__ void __launch_bounds__(256)
fa2_bwd_dq_finalize_kernel(const float* __restrict__ acc, uint16_t* __restrict__ dq, int N, int n_pad,
                           int d, long long groups8, int skip_rows, float scale) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= groups8) return;
    const long long e = i * 8;                            // element of dq, [BH][N][d]
    const long long row = e / d;
    const int col = static_cast<int>(e - row * d);
    const long long bh = row / N;
    const int n = static_cast<int>(row - bh * N);
    if (n < skip_rows) return;
    const float* src = acc + (bh * n_pad + n) * static_cast<long long>(d) + col;
    const float4 a = *reinterpret_cast<const float4*>(src);
    const float4 b = *reinterpret_cast<const float4*>(src + 4);
    uint4 w;
    if constexpr (F16) {
        w.x = ptx::pack_f16x2(a.x * scale, a.y * scale);
        w.y = ptx::pack_f16x2(a.z * scale, a.w * scale);
        w.z = ptx::pack_f16x2(b.x * scale, b.y * scale);
        w.w = ptx::pack_f16x2(b.z * scale, b.w * scale);
    } else {
        w.x = ptx::pack_bf16x2(a.x * scale, a.y * scale);
        w.y = ptx::pack_bf16x2(a.z * scale, a.w * scale);
        w.z = ptx::pack_bf16x2(b.x * scale, b.y * scale);
        w.w = ptx::pack_bf16x2(b.z * scale, b.w * scale);
    }
    *reinterpret_cast<uint4*>(dq + e) = w;
}

}  // namespace fa2
