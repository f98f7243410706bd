// fa2_fwd.cuh -- FlashAttention-2 forward kernel for sm_100a.
//
// Computes, for one 128-row query tile Q_i of one head (CS336 A2 Systems
// handout section 4.2.2, Algorithm 1):
//   for each key/value tile j:   S = scale * Q_i K_j^T            (step 9)
//                                m_new = max(m, rowmax S)         (step 10)
//                                P~ = exp(S - m_new)              (step 11)
//                                l = exp(m - m_new) l + rowsum P~ (step 12)
//                                O = diag(exp(m - m_new)) O + P~ V_j (step 13)
//   O = O / l,  L = m + log l                                      (steps 15-18)
// with the causal rule of Problem flash_forward (c): key tiles entirely above
// the diagonal are skipped, and on the diagonal tile scores of keys after the
// query are excluded (set to -inf, which is what the handout's -1e6 offset
// amounts to once exponentiated).
//
// The kernel serves fp32 inputs (TF32 MMAs) from d = 64 up; the library runs
// it at d = 80 and 128, where two fp32 query tiles per CTA (fa2_fwd2.cuh, which
// also serves every 16-bit input) leave too little shared memory.
//
// B200 mapping (one CTA per (query tile, head); 8 warps, warp-specialised):
//   warp 0    TMA producer: Q_i once, then K_j and V_j into two rings of
//             shared-memory stages guarded by full/empty mbarriers.
//   warp 1    MMA issuer (one thread): S_j = Q_i K_j^T into one of two
//             tensor-memory (TMEM) score buffers; O += P_j V_j with P_j read
//             from TMEM and O accumulated in TMEM (fp32).  Completion is
//             signalled with tcgen05.commit on mbarriers.
//   warps 2-5 softmax warpgroup: thread t owns query row t (TMEM lane t).  It
//             loads its score row from TMEM, applies the mask, updates the
//             running max / sum, writes P (fp32 rounded to TF32) back into
//             the score buffer for the next MMA, and rescales its O
//             row in TMEM when the running max grows.  After the last tile it
//             normalises O, stages it in shared memory for a TMA store and
//             writes L.
//   warps 6-7 operand rounding, warp 6 for Q and the K tiles, warp 7 for the
//             V tiles: rounds each tile in shared memory to TF32 (round to
//             nearest) once its TMA copy has landed and only then releases it
//             to the MMA issuer, so
//             the tensor core reads the operands exactly instead of dropping
//             their 13 low bits (a biased error); the softmax group rounds P
//             the same way.  The backward pass rounds its copies identically,
//             so its recomputed scores equal these.
// Scores are kept in log2 units (scale * log2(e) folded into one multiply)
// so every exponential is a single ex2.  The running max used as the
// exponent's reference is only raised when the row max grows by more than
// 2^8, which keeps P <= 256 and skips most O rescales; the final O / l and L
// are exact whatever reference was used.
#pragma once

#include <cstdint>

#include "fa2_traits.cuh"

namespace fa2 {

struct FwdParams {
    float* lse;            // [BH][N] natural-log logsumexp
    uint32_t* status;      // device status word
    int N;                 // query sequence length
    int Nk;                // key/value sequence length
    int BH;                // batch * heads
    int n_tiles;           // ceil(N / 128): query tiles
    int n_tiles_k;         // ceil(Nk / 128): key tiles
    int H, H_kv, group;    // query heads, key/value heads, H / H_kv
    int causal;
    float scale_log2;      // scale * log2(e)
    unsigned long long timeout_ns;
    const uint8_t* block_mask;  // [n_tiles][n_tiles_k] block mask, or nullptr (dense)
    const float* q32;      // fp32 inputs at d = 128: q itself, [BH][N][D] (read row by row)
    int head_group;        // two-tile forward: heads per group of work items (grouped_item)
    int one_tile;          // two-tile forward: one query tile per CTA (small grids)
};

template <int ES, int D>
struct FwdCfg {
    using G = TileGeom<ES, D>;
    // Q / K and V are rounded by separate warps (measured 1.45x at d = 128 and
    // 1.08x at d = 64 against one rounding warp).
    static constexpr int kThreads = 256;
    static constexpr int kBudget = 227 * 1024 - 2048;
    // fp32 at d = 128: Q sits in tensor memory (columns 384-511, beside the two
    // score buffers and O), written there rounded by the softmax threads; S =
    // Q K^T reads its A operand from TMEM, and the 64 KB of shared memory this
    // frees gives K a second ring stage.
    static constexpr bool kQInTmem = D == 128;
    static constexpr uint32_t kQCol = 384;
    static constexpr int kQBytes = kQInTmem ? 0 : G::kTileBytesK;   // Q staged in shared memory
    static constexpr int kFree = kBudget - kQBytes;
    // Ring depths for K and V (at most 4 each), as many as fit.
    static constexpr int kKV = G::kTileBytesK + G::kTileBytesMN;
    static constexpr int kPairs = kFree / kKV;
    static constexpr int kKSt0 = kPairs > 4 ? 4 : kPairs;
    static constexpr int kKSt = (kKSt0 < 4 && kFree - kKSt0 * kKV >= G::kTileBytesK) ? kKSt0 + 1 : kKSt0;
    static constexpr int kVSt = kKSt0;
    static_assert(kVSt >= 1, "shared memory too small for one K/V stage");
    static constexpr int kSmemBytes =
        1024 + kQBytes + G::kTileBytesK * kKSt + G::kTileBytesMN * kVSt;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kOCol = 256;
    // fp32 at d = 128, where one V stage is all that fits: K and V move through
    // their rings in parts, each with its own full / ready / empty barriers (K:
    // one 32-column box; V: four quarters of 32 keys), so a part is loaded,
    // rounded and fed to its MMAs while the next one is still on its way;
    // whole-tile hand-offs left the tensor pipe idle while each 64 KB tile was
    // loaded and rounded.  At d <= 80 the parts' extra waits cost more than they
    // overlap (measured 16 % slower at d = 64, 15 % at d = 80).
    static constexpr bool kParted = D == 128;
    static constexpr int kKParts = kParted ? G::kNBoxK : 1;
    static constexpr int kVParts = kParted ? 4 : 1;   // 4 measured 3-4 % faster than 2, 7 % than 1
    static constexpr int kKPartBytes = G::kTileBytesK / kKParts;
    static constexpr int kVPartBytes = G::kTileBytesMN / kVParts;
    static constexpr int kVPartRows = kTileRows / kVParts;
    static constexpr int kKStepsPart = kParted ? G::kBoxK / G::kKStep : G::kStepsD;  // QK^T steps per K part
    static constexpr int kVStepsPart = G::kStepsRows / kVParts;                          // PV steps per V part
    static_assert(kKParts * kKStepsPart >= G::kStepsD, "K parts miss a contraction step");
    static_assert(kVParts * kVStepsPart == G::kStepsRows, "V parts miss a contraction step");
};

// Rounds BYTES bytes of fp32 values in shared memory to TF32 in place (one
// warp), then makes the writes visible to the tensor core's operand reads.
// BATCHED (fp32, d >= 64): batches of eight 16-byte loads per lane, so the
// warp runs near shared-memory bandwidth instead of one load latency per
// vector; otherwise the plain strided loop (the batched form, and a fully
// unrolled one, measured 10-40 % slower at d <= 32).
template <int BYTES, bool BATCHED>
__device__ __forceinline__ void round_tf32_smem(uint8_t* base, int lane) {
    float4* p4 = reinterpret_cast<float4*>(base);
    auto rna = [](float4 x) {
        x.x = __uint_as_float(ptx::to_tf32_rna(x.x));
        x.y = __uint_as_float(ptx::to_tf32_rna(x.y));
        x.z = __uint_as_float(ptx::to_tf32_rna(x.z));
        x.w = __uint_as_float(ptx::to_tf32_rna(x.w));
        return x;
    };
    if constexpr (BATCHED) {
        constexpr int kUnroll = 8;
        static_assert(BYTES % (16 * 32 * kUnroll) == 0, "tile not a whole number of rounding batches");
#pragma unroll 1
        for (int b = 0; b < BYTES / (16 * 32 * kUnroll); ++b) {
            float4 x[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) x[u] = p4[(b * kUnroll + u) * 32 + lane];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) p4[(b * kUnroll + u) * 32 + lane] = rna(x[u]);
        }
    } else {
        for (int i = lane; i < BYTES / 16; i += 32) p4[i] = rna(p4[i]);
    }
    ptx::fence_async_smem();
    __syncwarp();
}

template <int ES, int D, bool SPARSE = false>
__global__ void __launch_bounds__(FwdCfg<ES, D>::kThreads, 1)
fa2_fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
               const FwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = FwdCfg<ES, D>;
    using G = typename Cfg::G;
    static_assert(ES == 4 && D >= 64, "the one-tile kernel serves fp32 inputs from d = 64 up");
    constexpr int KST = Cfg::kKSt;
    constexpr int VST = Cfg::kVSt;
    constexpr int KP = Cfg::kKParts;
    constexpr int VP = Cfg::kVParts;
    constexpr int KS = KST * KP;       // K part slots: part b of stage ks is slot ks * KP + b
    constexpr int VS = VST * VP;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_q_full;
    __shared__ uint64_t bar_k_full[KS], bar_k_empty[KS];
    __shared__ uint64_t bar_v_full[VS], bar_v_empty[VS];
    __shared__ uint64_t bar_s_full[2], bar_p_full[2], bar_o_done, bar_drain;
    // Tiles released by the rounding warps (the MMA issuer waits on these).
    __shared__ uint64_t bar_q_ready, bar_k_ready[KS], bar_v_ready[VS];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    __shared__ int s_cnt;                      // block-sparse: key tiles of this query tile
    uint64_t* const q_go = &bar_q_ready;
    uint64_t* const k_go = bar_k_ready;
    uint64_t* const v_go = bar_v_ready;

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    constexpr bool QT = Cfg::kQInTmem;
    uint8_t* sQ = smem;                        // unused when Q is in tensor memory
    uint8_t* sK = sQ + Cfg::kQBytes;
    // O is staged for its store in the Q slot, or in K stage 0 (idle by then).
    uint8_t* sO = QT ? sK : sQ;
    uint8_t* sV = sK + KST * G::kTileBytesK;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: causal query tiles are issued longest first.
    const int item = blockIdx.x;
    const int tile_rank = item / p.BH;
    const int bh = item - tile_rank * p.BH;
    const int q_tile = p.causal ? (p.n_tiles - 1 - tile_rank) : tile_rank;
    // Key tiles this query tile sees (causal: key index <= query index); with a
    // block mask, those whose block is set, found by each thread walking the
    // mask row (no shared-memory list here: the fp32 tiles fill shared memory).
    const int n_kv_lim = p.causal ? min(q_tile + 1, p.n_tiles_k) : p.n_tiles_k;
    const int q_row0 = q_tile * kTileRows;
    const int bh_kv = kv_head_of(bh, p.H, p.H_kv, p.group);
    const uint8_t* mask_row = SPARSE ? p.block_mask + static_cast<size_t>(q_tile) * p.n_tiles_k : nullptr;
    auto blk_set = [&](int j) { return __ldg(mask_row + j) != 0; };
    if (SPARSE && warp == 0) {
        int c = 0;
        for (int base = 0; base < n_kv_lim; base += 32)
            c += __popc(__ballot_sync(0xffffffffu, base + lane < n_kv_lim && blk_set(base + lane)));
        if (lane == 0) s_cnt = c;
    }

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_q_full, 1);
        for (int s = 0; s < KS; ++s) { ptx::mbar_init(&bar_k_full[s], 1); ptx::mbar_init(&bar_k_empty[s], 1); }
        for (int s = 0; s < VS; ++s) { ptx::mbar_init(&bar_v_full[s], 1); ptx::mbar_init(&bar_v_empty[s], 1); }
        for (int b = 0; b < 2; ++b) { ptx::mbar_init(&bar_s_full[b], 1); ptx::mbar_init(&bar_p_full[b], 4); }
        ptx::mbar_init(&bar_q_ready, QT ? 4 : 1);   // QT: one arrival per softmax warp
        for (int s = 0; s < KS; ++s) ptx::mbar_init(&bar_k_ready[s], 1);
        for (int s = 0; s < VS; ++s) ptx::mbar_init(&bar_v_ready[s], 1);
        ptx::mbar_init(&bar_o_done, 1);
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
    const int n_kv = SPARSE ? s_cnt : n_kv_lim;
    MaskWalk walker;
    auto kv_of = [&](int j) { return SPARSE ? walker.at(j, n_kv_lim, blk_set) : j; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // (nothing for a query tile without key tiles: its epilogue stages zeros
        // in the Q slot, which no copy or rounding may touch then)
        if (lane == 0 && n_kv > 0) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            if (!QT) {
                ptx::mbar_arrive_expect_tx(&bar_q_full, G::kTileBytesK);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sQ + b * kTileRows * G::kRowBK, &tm_q, &bar_q_full, b * G::kBoxK, q_row0, bh);
            }
            // K parts and V parts are issued as their slots free up, each ring on
            // its own (a V slot still in use does not hold back the next K part).
            MaskWalk walk_k, walk_v;
            const int k_tot = n_kv * KP, v_tot = n_kv * VP;
            int kn = 0, vn = 0;                     // parts issued
            uint32_t spins = 0;
            uint64_t t_idle = 0;
            while (kn < k_tot || vn < v_tot) {
                bool moved = false;
                if (kn < k_tot) {
                    const int j = kn / KP, b = kn - j * KP, sl = (j % KST) * KP + b;
                    if (j < KST || ptx::mbar_test_wait(&bar_k_empty[sl], ((j / KST) & 1) ^ 1)) {
                        const int kv = SPARSE ? walk_k.at(j, n_kv_lim, blk_set) : j;
                        uint8_t* dk = sK + (j % KST) * G::kTileBytesK;
                        constexpr int kBoxes = G::kNBoxK / KP;
                        ptx::mbar_arrive_expect_tx(&bar_k_full[sl], Cfg::kKPartBytes);
                        for (int bb = b * kBoxes; bb < (b + 1) * kBoxes; ++bb)
                            ptx::tma_load_3d(dk + bb * kTileRows * G::kRowBK, &tm_k, &bar_k_full[sl], bb * G::kBoxK, kv * kTileRows, bh_kv);
                        ++kn;
                        moved = true;
                    }
                }
                if (vn < v_tot) {
                    const int j = vn / VP, h = vn - j * VP, sl = (j % VST) * VP + h;
                    if (j < VST || ptx::mbar_test_wait(&bar_v_empty[sl], ((j / VST) & 1) ^ 1)) {
                        const int kv = SPARSE ? walk_v.at(j, n_kv_lim, blk_set) : j;
                        uint8_t* dv = sV + (j % VST) * G::kTileBytesMN + h * Cfg::kVPartBytes;
                        ptx::mbar_arrive_expect_tx(&bar_v_full[sl], Cfg::kVPartBytes);
                        for (int c = 0; c < G::kNBoxMN; ++c)
                            ptx::tma_load_3d(dv + c * Cfg::kVPartRows * G::kRowBMN, &tm_v, &bar_v_full[sl], c * G::kBoxMN,
                                             kv * kTileRows + h * Cfg::kVPartRows, bh_kv);
                        ++vn;
                        moved = true;
                    }
                }
                if (moved) {
                    spins = 0;
                } else if (spins++ == 0) {
                    t_idle = ptx::globaltimer_ns();
                } else if ((spins & 63u) == 0) {
                    // Bounded, as every wait here: give up on abort or after the timeout.
                    if (abort_flag) break;
                    if (ptx::globaltimer_ns() - t_idle > tmo) { abort_flag = 1u; break; }
                }
            }
            if (abort_flag) {
                // Let copies already in flight land before the CTA exits.
                constexpr uint64_t kDrainNs = 20000000ull;
                if (!QT) ptx::mbar_wait_drain(&bar_q_full, 0, kDrainNs);
                for (int t = kn - 1; t >= 0 && t >= kn - KS; --t)
                    ptx::mbar_wait_drain(&bar_k_full[((t / KP) % KST) * KP + t % KP], ((t / KP) / KST) & 1, kDrainNs);
                for (int t = vn - 1; t >= 0 && t >= vn - VS; --t)
                    ptx::mbar_wait_drain(&bar_v_full[((t / VP) % VST) * VP + t % VP], ((t / VP) / VST) & 1, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n_kv > 0) {
            constexpr uint32_t idesc_qk = ptx::instr_desc(G::kFmt, 128, 128, false, false);
            constexpr uint32_t idesc_pv = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            const uint32_t q_addr = ptx::smem_addr(sQ);
            bool ok = ptx::mbar_wait(q_go, 0, &abort_flag, tmo);
            auto issue_pv = [&](int jj) -> bool {
                if (!ptx::mbar_wait(&bar_p_full[jj & 1], (jj >> 1) & 1, &abort_flag, tmo)) return false;
                const int vs = jj % VST;
                const uint32_t p_tmem = tmem + (jj & 1) * 128;
                for (int h = 0; h < VP; ++h) {
                    const int sl = vs * VP + h;
                    if (!ptx::mbar_wait(&v_go[sl], (jj / VST) & 1, &abort_flag, tmo)) return false;
                    ptx::tc_fence_after();
                    const uint32_t v_addr = ptx::smem_addr(sV + vs * G::kTileBytesMN + h * Cfg::kVPartBytes);
#pragma unroll
                    for (int k2 = 0; k2 < Cfg::kVStepsPart; ++k2) {
                        const int kk = h * Cfg::kVStepsPart + k2;
                        const uint64_t bdesc = desc_mnmajor<G>(v_addr, k2, Cfg::kVPartRows);
                        ptx::mma_tf32_ts(tmem + Cfg::kOCol, p_tmem + kk * 8, bdesc, idesc_pv, (jj > 0 || kk > 0) ? 1u : 0u);
                    }
                    ptx::mma_commit(&bar_v_empty[sl]);
                }
                ptx::mma_commit(&bar_o_done);
                return true;
            };
            for (int j = 0; ok && j < n_kv; ++j) {
                const int ks = j % KST;
                const uint32_t k_addr = ptx::smem_addr(sK + ks * G::kTileBytesK);
                const uint32_t s_tmem = tmem + (j & 1) * 128;
                for (int b = 0; b < KP; ++b) {
                    const int sl = ks * KP + b;
                    if (!ptx::mbar_wait(&k_go[sl], (j / KST) & 1, &abort_flag, tmo)) { ok = false; break; }
                    ptx::tc_fence_after();
#pragma unroll
                    for (int k2 = 0; k2 < Cfg::kKStepsPart; ++k2) {
                        const int kk = b * Cfg::kKStepsPart + k2;
                        if (kk < G::kStepsD) {
                            const uint64_t bdesc = desc_kmajor<G>(k_addr, kk);
                            if constexpr (QT)
                                ptx::mma_tf32_ts(s_tmem, tmem + Cfg::kQCol + kk * G::kKStep, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                            else
                                ptx::mma_tf32_ss(s_tmem, desc_kmajor<G>(q_addr, kk), bdesc, idesc_qk, kk > 0 ? 1u : 0u);
                        }
                    }
                    ptx::mma_commit(&bar_k_empty[sl]);
                }
                if (!ok) break;
                ptx::mma_commit(&bar_s_full[j & 1]);
                if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
            }
            if (ok) ok = issue_pv(n_kv - 1);
            if (!ok) {
                // Drain: every MMA issued so far must finish before TMEM is freed.
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else if (warp < 6) {
        // ------------------------------------------------ softmax warpgroup
        const int quarter = warp & 3;           // TMEM lane quarter this warp may access
        const int r = quarter * 32 + lane;      // query row inside the tile
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const uint32_t o_tmem = lane_base + Cfg::kOCol;
        const float sl2 = p.scale_log2;
        float m_ref = -INFINITY;                // reference max (log2 units)
        float l = 0.f;                          // running sum of 2^(t - m_ref)
        bool ok = true;
        if constexpr (QT) {
            // Query row r, rounded to TF32, into tensor memory; zeros past N.
            if (n_kv > 0) {
                const bool row_valid = q_row0 + r < p.N;
                const float4* src = reinterpret_cast<const float4*>(
                    p.q32 + (static_cast<size_t>(bh) * p.N + (row_valid ? q_row0 + r : 0)) * D);
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t u[32];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 x = row_valid ? __ldg(src + c0 / 4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
                        u[4 * q4 + 0] = ptx::to_tf32_rna(x.x);
                        u[4 * q4 + 1] = ptx::to_tf32_rna(x.y);
                        u[4 * q4 + 2] = ptx::to_tf32_rna(x.z);
                        u[4 * q4 + 3] = ptx::to_tf32_rna(x.w);
                    }
                    ptx::tmem_st32(lane_base + Cfg::kQCol + c0, u);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_q_ready);
            }
        }
        for (int j = 0; j < n_kv; ++j) {
            if (!ptx::mbar_wait(&bar_s_full[j & 1], (j >> 1) & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t s_tmem = lane_base + (j & 1) * 128;
            float s[128];
            {
                uint32_t u[32];
#pragma unroll
                for (int c0 = 0; c0 < 128; c0 += 32) {
                    ptx::tmem_ld32(s_tmem + c0, u);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) s[c0 + c] = __uint_as_float(u[c]);
                }
            }
            // Mask: causal diagonal tile (key > query), or keys past N.
            const int kv = kv_of(j);
            const bool diag = p.causal && (kv == q_tile);
            const int kv_valid = p.Nk - kv * kTileRows;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                float t = s[c] * sl2;
                if ((diag && c > r) || c >= kv_valid) t = -INFINITY;
                s[c] = t;
                mx = fmaxf(mx, t);
            }
            const float m_new = fmaxf(m_ref, mx);
            float alpha = 1.f;
            const bool raise = (m_new - m_ref) > 8.f;   // true on the first tile
            if (raise) {
                alpha = ptx::ex2_approx(m_ref - m_new);
                m_ref = m_new;
            }
            if (j > 0) {
                // PV_{j-1} must be done before O is touched.
                if (!ptx::mbar_wait(&bar_o_done, (j - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
                    for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                        uint32_t u[16];
                        ptx::tmem_ld16(o_tmem + c0, u);
                        ptx::tmem_wait_ld();
#pragma unroll
                        for (int c = 0; c < 16; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
                        ptx::tmem_st16(o_tmem + c0, u);
                    }
                }
            }
            l *= alpha;
            float rs = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                const float pc = ptx::ex2_approx(s[c] - m_ref);
                s[c] = pc;
                rs += pc;
            }
            l += rs;
            // P, rounded to TF32, back into the score buffer (A operand of the PV MMA).
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32) {
                uint32_t u[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) u[c] = ptx::to_tf32_rna(s[c0 + c]);
                ptx::tmem_st32(s_tmem + c0, u);
            }
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_p_full[j & 1]);
        }
        // ---------------- epilogue: O / l -> shared memory -> TMA store; L.  A query
        // tile whose block row is empty writes O = 0 and L = -inf.
        if (ok && n_kv > 0) ok = ptx::mbar_wait(&bar_o_done, (n_kv - 1) & 1, &abort_flag, tmo);
        if (ok) {
            ptx::tc_fence_after();
            const float inv_l = n_kv > 0 ? 1.f / l : 0.f;
#pragma unroll
            for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                uint32_t u[16] = {};
                if (n_kv > 0) {
                    ptx::tmem_ld16(o_tmem + c0, u);
                    ptx::tmem_wait_ld();
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int col = c0 + 4 * q4;
                    if (col < D) {
                        uint4 w;
                        w.x = __float_as_uint(__uint_as_float(u[4 * q4 + 0]) * inv_l);
                        w.y = __float_as_uint(__uint_as_float(u[4 * q4 + 1]) * inv_l);
                        w.z = __float_as_uint(__uint_as_float(u[4 * q4 + 2]) * inv_l);
                        w.w = __float_as_uint(__uint_as_float(u[4 * q4 + 3]) * inv_l);
                        *reinterpret_cast<uint4*>(sO + kmajor_chunk_offset<G>(r, col)) = w;
                    }
                }
            }
            const int q_row = q_row0 + r;
            if (q_row < p.N)
                p.lse[static_cast<size_t>(bh) * p.N + q_row] =
                    n_kv > 0 ? (m_ref + __log2f(l)) * 0.69314718055994531f : -INFINITY;
            ptx::fence_async_smem();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok && threadIdx.x == 64) {
            for (int b = 0; b < G::kNBoxK; ++b)
                ptx::tma_store_3d(&tm_o, sO + b * kTileRows * G::kRowBK, b * G::kBoxK, q_row0, bh);
            ptx::tma_store_commit();
            ptx::tma_store_wait_all();
        }
    } else {
        // ------------------------------------------------ TF32 rounding
        if (warp == 6) {
            // Q (unless it is in tensor memory) and the K parts.
            bool ok = n_kv > 0 && (QT || ptx::mbar_wait(&bar_q_full, 0, &abort_flag, tmo));
            if (ok && !QT) {
                round_tf32_smem<G::kTileBytesK, true>(sQ, lane);
                if (lane == 0) ptx::mbar_arrive(&bar_q_ready);
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const int ks = j % KST;
                for (int b = 0; ok && b < KP; ++b) {
                    if (!ptx::mbar_wait(&bar_k_full[ks * KP + b], (j / KST) & 1, &abort_flag, tmo)) { ok = false; break; }
                    round_tf32_smem<Cfg::kKPartBytes, true>(sK + ks * G::kTileBytesK + b * Cfg::kKPartBytes, lane);
                    if (lane == 0) ptx::mbar_arrive(&bar_k_ready[ks * KP + b]);
                }
            }
        } else {
            // The V parts.
            bool ok = true;
            for (int j = 0; ok && j < n_kv; ++j) {
                const int vs = j % VST;
                for (int h = 0; h < VP; ++h) {
                    if (!ptx::mbar_wait(&bar_v_full[vs * VP + h], (j / VST) & 1, &abort_flag, tmo)) { ok = false; break; }
                    round_tf32_smem<Cfg::kVPartBytes, true>(sV + vs * G::kTileBytesMN + h * Cfg::kVPartBytes, lane);
                    if (lane == 0) ptx::mbar_arrive(&bar_v_ready[vs * VP + h]);
                }
            }
        }
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
