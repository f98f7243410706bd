// fa2_fwd2.cuh -- FlashAttention-2 forward for sm_100a, two query tiles per CTA.
//
// Same computation as fa2_fwd.cuh (CS336 A2 Systems handout section 4.2.2,
// Algorithm 1, with the causal rule of Problem flash_forward (c)), organised so
// that the exponentials of one query tile overlap the tensor-core work of the
// other:
//
//   warp 0     TMA producer: Q_A and Q_B (two adjacent 128-row query tiles of
//              one head) once, then K_j / V_j through rings of shared-memory
//              stages.
//   warp 1     MMA issuer (one thread).  Per key tile j it issues, in order,
//                PV_A(j-1) -> S_A(j) ... as soon as each operand is ready:
//                  O_A += P_A(j) V_j ; S_A(j+1) = Q_A K_{j+1}^T ;
//                  O_B += P_B(j) V_j ; S_B(j+1) = Q_B K_{j+1}^T
//              so while softmax warpgroup A works on S_A(j+1) the tensor core
//              runs PV_B(j) and S_B(j+1), and the other way round.
//   warp 2     load watcher: adds the arrival that tells the issuer V_j and
//              K_{j+1} have landed to the P-ready barrier, so the issuer waits
//              on that barrier alone.
//   warp 3     fp32 inputs: rounds each landed Q, K and V tile to TF32 in
//              shared memory (round to nearest, as the one-tile kernel and the
//              backward's operand copies do) and only then releases it; the
//              issuer and the watcher wait on those releases.  Idle otherwise.
//   warps 4-7  softmax warpgroup for tile A; warps 8-11 for tile B.  Thread t
//              owns query row t of its tile (tensor-memory lane t).
//   Warpgroup 0 (warps 0-3) runs with fewer registers and the softmax
//   warpgroups with more (setmaxnreg), so the score rows fit without spills.
//
// Tensor memory (512 columns): S_A | S_B | O_A | O_B, 128 columns each; P is
// written over its S buffer (bf16 pairs, or fp32 for the TF32 path) and read
// by the PV MMA as its A operand.
//
// Per-row arithmetic: the running max is kept on raw scores (scale > 0), so
// each exponent is one fused multiply-add feeding ex2:
//   p = 2^(s * scale*log2(e) - m * scale*log2(e)).
// The reference max is raised only when a row's max grows by more than 2^8 in
// the exponent (then O and l are rescaled); O / l and L are exact for any
// reference.
#pragma once

#include <cstdint>

#include "fa2_traits.cuh"
#include "fa2_fwd.cuh"

namespace fa2 {

template <int ES, int D, bool F16 = false>
struct Fwd2Cfg {
    using G = TileGeom<ES, D, F16>;
    // Warpgroup 0: warp 0 TMA producer, 1 MMA issuer, 2 load watcher, 3 idle;
    // warpgroups 1 / 2 (warps 4-7 / 8-11): softmax of query tile A / B.
    static constexpr int kThreads = 384;
    // Twelve warps put three on each SM sub-partition, so a thread starts with
    // (16384 / 96) rounded down to a multiple of 8 = 168 registers.  Warpgroup
    // 0 gives registers back (setmaxnreg.dec) and the softmax warpgroups, which
    // hold a whole 128-column fp32 score row, take them (setmaxnreg.inc); the
    // split must fit in what the block was launched with.
    static constexpr int kLaunchRegs = 168;
    static constexpr int kRegsLow = 72;
    static constexpr int kRegsHigh = 216;
    static_assert(128 * kRegsLow + 256 * kRegsHigh <= kThreads * kLaunchRegs,
                  "register split exceeds the registers the block is launched with");
    static_assert(kRegsLow % 8 == 0 && kRegsHigh % 8 == 0 && kRegsLow >= 24 && kRegsHigh <= 256,
                  "setmaxnreg counts are multiples of 8 in [24, 256]");
    static constexpr int kBudget = 227 * 1024 - 2048;
    static constexpr int kQBytes = 2 * G::kTileBytesK;
    static constexpr int kFree = kBudget - kQBytes;
    static constexpr int kKV = G::kTileBytesK + G::kTileBytesMN;
    static constexpr int kPairs = kFree / kKV;
    static constexpr int kStages = kPairs > 4 ? 4 : kPairs;
    static constexpr bool kFits = kPairs >= 1;
    static constexpr int kSmemBytes = 1024 + kQBytes + (kStages > 0 ? kStages : 1) * kKV;
    static constexpr uint32_t kTmemCols = 512;
    // TMEM columns of tile t's score buffer and output accumulator.
    static __device__ __forceinline__ uint32_t col_s(int t) { return 128u * t; }
    static __device__ __forceinline__ uint32_t col_o(int t) { return 256u + 128u * t; }
};

// Block-sparse: the mask rows of a CTA's two query tiles, and the largest key
// tile each may see (causal limit; -1 for a missing tile B).
struct PairRows {
    const uint8_t* row[2];
    int lim[2];
    __device__ __forceinline__ bool on(int t, int j) const { return j <= lim[t] && __ldg(row[t] + j) != 0; }
    __device__ __forceinline__ bool any(int j) const { return on(0, j) || on(1, j); }
};

// One softmax warpgroup: processes query tile `t` (0 = A, 1 = B) for key
// tiles 0 .. n_kv-1 (block-sparse: its own n_kv set blocks), then writes its O
// tile and L rows.
template <int ES, int D, bool F16, bool SPARSE>
__device__ __forceinline__ void fwd2_softmax(const FwdParams p, int t, int q_tile, int n_kv,
                                             int bh, uint32_t tmem, uint8_t* sQt,
                                             uint64_t* bar_s_full, uint64_t* bar_p_full,
                                             uint64_t* bar_o_done, const PairRows* pr,
                                             volatile uint32_t* abort_flag,
                                             const CUtensorMap* tm_o) {
    using Cfg = Fwd2Cfg<ES, D, F16>;
    using G = typename Cfg::G;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
    const uint32_t s_tmem = lane_base + Cfg::col_s(t);
    const uint32_t o_tmem = lane_base + Cfg::col_o(t);
    const uint64_t tmo = p.timeout_ns;
    const float sl2 = p.scale_log2;
    const int q_row0 = q_tile * kTileRows;
    float m_raw = -INFINITY;    // reference max of raw scores
    float l = 0.f;
    bool ok = true;
    MaskWalk walker;
    for (int j = 0; j < n_kv; ++j) {
        // Key tile of step j, and (block-sparse) whether its block is set for this
        // query tile: a step the other tile needs but this one does not is masked.
        // (block-sparse: step j is the j-th key tile whose block is set for this
        // query tile; the pair's other tile may take steps in between)
        int kv = j;
        const bool blk_on = true;
        if constexpr (SPARSE) kv = walker.at(j, p.n_tiles_k, [&](int x) { return pr->on(t, x); });
        if (!ptx::mbar_wait(bar_s_full, j & 1, abort_flag, tmo)) { ok = false; break; }
        ptx::tc_fence_after();
        float s[128];
        {
            uint32_t u[128];
#pragma unroll
            for (int c0 = 0; c0 < 128; c0 += 32)
                ptx::tmem_ld32(s_tmem + c0, *reinterpret_cast<uint32_t(*)[32]>(u + c0));
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = __uint_as_float(u[c]);
        }
        const int kv_valid = p.Nk - kv * kTileRows;
        if (SPARSE && !blk_on) {
#pragma unroll
            for (int c = 0; c < 128; ++c) s[c] = -INFINITY;
        }
        if (p.causal && kv == q_tile) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (c > r) s[c] = -INFINITY;
        }
        if (kv_valid < kTileRows) {
#pragma unroll
            for (int c = 0; c < 128; ++c)
                if (c >= kv_valid) s[c] = -INFINITY;
        }
        float mx0 = s[0], mx1 = s[1];
#pragma unroll
        for (int c = 2; c < 126; c += 4) {
            mx0 = ptx::max3(mx0, s[c], s[c + 1]);
            mx1 = ptx::max3(mx1, s[c + 2], s[c + 3]);
        }
        const float mx = ptx::max3(mx0, mx1, fmaxf(s[126], s[127]));
        const float m_new = fmaxf(m_raw, mx);
        const bool raise = (m_new - m_raw) * sl2 > 8.f;   // true on the first tile
        float alpha = 1.f;
        if (raise) {
            alpha = ptx::ex2_approx((m_raw - m_new) * sl2);
            m_raw = m_new;
        }
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
            // PV(j-1) must have finished before O is rescaled.
            if (!ptx::mbar_wait(bar_o_done, (j - 1) & 1, abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
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
        l *= alpha;
        // Until the row has seen a key (block-sparse: leading masked steps) the
        // reference max is -inf; exponentiate against 0 so masked scores give 0.
        const float neg = (SPARSE && m_raw == -INFINITY) ? 0.f : -m_raw * sl2;
        const float2 sl2v = make_float2(sl2, sl2), negv = make_float2(neg, neg);
        float2 rs = make_float2(0.f, 0.f);      // even / odd column sums
        // Exponentiate 32 columns at a time and store them as P right away.
#pragma unroll
        for (int c0 = 0; c0 < 128; c0 += 32) {
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
                const float2 a = ptx::fma2(make_float2(s[c0 + c], s[c0 + c + 1]), sl2v, negv);
                s[c0 + c] = ptx::ex2_approx(a.x);
                s[c0 + c + 1] = ptx::ex2_approx(a.y);
                rs = ptx::add2(rs, make_float2(s[c0 + c], s[c0 + c + 1]));
            }
            if constexpr (G::kF32) {
                uint32_t u[32];
#pragma unroll
                for (int c = 0; c < 32; ++c) u[c] = ptx::to_tf32_rna(s[c0 + c]);
                ptx::tmem_st32(s_tmem + c0, u);
            } else {
                uint32_t u[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) u[c] = G::pack2(s[c0 + 2 * c], s[c0 + 2 * c + 1]);
                ptx::tmem_st16(s_tmem + c0 / 2, u);
            }
        }
        l += rs.x + rs.y;
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar_p_full);
    }
    // ---------------- epilogue: O / l -> shared memory (this tile's Q slot) -> TMA.
    // A row that saw no key (l = 0: an empty or fully masked block row) gets O = 0
    // and L = -inf; a tile with no key step writes that without touching TMEM.
    if (ok && (!SPARSE || n_kv > 0)) ok = ptx::mbar_wait(bar_o_done, (n_kv - 1) & 1, abort_flag, tmo);
    if (ok) {
        ptx::tc_fence_after();
        const float inv_l = (!SPARSE || l > 0.f) ? 1.f / l : 0.f;
#pragma unroll
        for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
            uint32_t u[16];
            if (SPARSE && n_kv == 0) {
#pragma unroll
                for (int c = 0; c < 16; ++c) u[c] = 0u;
            } else {
                ptx::tmem_ld16(o_tmem + c0, u);
                ptx::tmem_wait_ld();
            }
            if constexpr (G::kF32) {
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const int col = c0 + 4 * q4;
                    if (col < D) {
                        uint4 w;
                        w.x = __float_as_uint(__uint_as_float(u[4 * q4 + 0]) * inv_l);
                        w.y = __float_as_uint(__uint_as_float(u[4 * q4 + 1]) * inv_l);
                        w.z = __float_as_uint(__uint_as_float(u[4 * q4 + 2]) * inv_l);
                        w.w = __float_as_uint(__uint_as_float(u[4 * q4 + 3]) * inv_l);
                        *reinterpret_cast<uint4*>(sQt + kmajor_chunk_offset<G>(r, col)) = w;
                    }
                }
            } else {
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const int col = c0 + 8 * h8;
                    if (col < D) {
                        uint4 w;
                        const float* f = reinterpret_cast<const float*>(u) + 8 * h8;
                        w.x = G::pack2(f[0] * inv_l, f[1] * inv_l);
                        w.y = G::pack2(f[2] * inv_l, f[3] * inv_l);
                        w.z = G::pack2(f[4] * inv_l, f[5] * inv_l);
                        w.w = G::pack2(f[6] * inv_l, f[7] * inv_l);
                        *reinterpret_cast<uint4*>(sQt + kmajor_chunk_offset<G>(r, col)) = w;
                    }
                }
            }
        }
        const int q_row = q_row0 + r;
        if (q_row < p.N)
            p.lse[static_cast<size_t>(bh) * p.N + q_row] =
                (m_raw * sl2 + __log2f(l)) * 0.69314718055994531f;
        ptx::fence_async_smem();
    }
    if (t == 0)
        asm volatile("bar.sync 1, 128;" ::: "memory");
    else
        asm volatile("bar.sync 2, 128;" ::: "memory");
    if (ok && (threadIdx.x & 127) == 0) {
        for (int b = 0; b < G::kNBoxK; ++b)
            ptx::tma_store_3d(tm_o, sQt + b * kTileRows * G::kRowBK, b * G::kBoxK, q_row0, bh);
        ptx::tma_store_commit();
        ptx::tma_store_wait_all();
    }
}

template <int ES, int D, bool F16 = false, bool SPARSE = false>
__global__ void __launch_bounds__(384, 1)
fa2_fwd2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                const FwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = Fwd2Cfg<ES, D, F16>;
    using G = typename Cfg::G;
    constexpr int ST = Cfg::kStages;
    static_assert(ST >= 1, "two query tiles and one K/V stage do not fit in shared memory");

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_q_full;
    __shared__ uint64_t bar_k_full[ST], bar_k_empty[ST], bar_v_full[ST], bar_v_empty[ST];
    __shared__ uint64_t bar_s_full[2], bar_p_full[2], bar_o_done[2], bar_drain;
    // fp32: tiles released by the rounding warp (what the issuer and watcher wait on).
    __shared__ uint64_t bar_q_ready, bar_k_ready[ST], bar_v_ready[ST];
    uint64_t* const q_go = G::kF32 ? &bar_q_ready : &bar_q_full;
    uint64_t* const k_go = G::kF32 ? bar_k_ready : bar_k_full;
    uint64_t* const v_go = G::kF32 ? bar_v_ready : bar_v_full;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    // Block-sparse: the pair's key tiles, in order, with bit 14 / 15 set when
    // the block of query tile A / B is set (the first kMaxMaskTiles steps);
    // s_cnt = set blocks of tile A, of tile B, of the pair.
    __shared__ uint16_t s_kv[SPARSE ? kMaxMaskTiles : 1];
    __shared__ int s_cnt[3];
    __shared__ PairRows s_pr;

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sQ[2] = {smem, smem + G::kTileBytesK};
    uint8_t* sK = smem + Cfg::kQBytes;
    uint8_t* sV = sK + ST * G::kTileBytesK;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: a pair of adjacent query tiles (2t, 2t+1) of one head, or (when
    // pairs would leave SMs idle, p.one_tile) a single query tile t with no
    // tile B; causal items are issued longest first.
    const int n_items = p.one_tile ? p.n_tiles : (p.n_tiles + 1) >> 1;
    int rank, bh;
    grouped_item(blockIdx.x, n_items, p.BH, p.head_group, rank, bh);
    const int pair = p.causal ? (n_items - 1 - rank) : rank;
    const int tile[2] = {p.one_tile ? pair : 2 * pair, p.one_tile ? p.n_tiles : 2 * pair + 1};
    const bool has_b = tile[1] < p.n_tiles;
    const int bh_kv = kv_head_of(bh, p.H, p.H_kv, p.group);
    constexpr bool sparse = SPARSE;
    // Key tiles of the pair: those whose block is set for tile A or tile B (and,
    // causal, at or below that tile).  The producer streams their union; each
    // tile takes MMAs and softmax steps for its own set blocks only.
    if (sparse && warp == 0) {
        PairRows pr;
        const int last = p.n_tiles_k - 1;
        pr.row[0] = p.block_mask + static_cast<size_t>(tile[0]) * p.n_tiles_k;
        pr.row[1] = p.block_mask + static_cast<size_t>(has_b ? tile[1] : tile[0]) * p.n_tiles_k;
        pr.lim[0] = p.causal ? min(tile[0], last) : last;
        pr.lim[1] = has_b ? (p.causal ? min(tile[1], last) : last) : -1;
        if (lane == 0) s_pr = pr;
        const int n_pair = warp_compact(s_kv, p.n_tiles_k, [&](int j) { return pr.any(j); },
            [&](int j) { return j | (pr.on(0, j) ? 0x4000 : 0) | (pr.on(1, j) ? 0x8000 : 0); });
        int own[2] = {0, 0};
        for (int base = 0; base < p.n_tiles_k; base += 32) {
            const int j = base + lane;
            own[0] += __popc(__ballot_sync(0xffffffffu, j < p.n_tiles_k && pr.on(0, j)));
            own[1] += __popc(__ballot_sync(0xffffffffu, j < p.n_tiles_k && pr.on(1, j)));
        }
        if (lane == 0) { s_cnt[0] = own[0]; s_cnt[1] = own[1]; s_cnt[2] = n_pair; }
    }

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_q_full, 1);
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&bar_k_full[s], 1);
            ptx::mbar_init(&bar_k_empty[s], 1);
            ptx::mbar_init(&bar_v_full[s], 1);
            ptx::mbar_init(&bar_v_empty[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            ptx::mbar_init(&bar_s_full[t], 1);
            // 4 softmax warps + the load watcher (block-sparse: the issuer checks
            // the loads itself)
            ptx::mbar_init(&bar_p_full[t], SPARSE ? 4 : 5);
            ptx::mbar_init(&bar_o_done[t], 1);
        }
        ptx::mbar_init(&bar_drain, 1);
        ptx::mbar_init(&bar_q_ready, 1);
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&bar_k_ready[s], 1);
            ptx::mbar_init(&bar_v_ready[s], 1);
        }
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
    // Key-tile steps each query tile takes (causal: key index <= query index;
    // dense: tile A's steps are a prefix of tile B's; block-sparse: each tile's
    // own set blocks) and the steps the producer streams (their union).
    int n_kv_t[2];
    if (sparse) {
        n_kv_t[0] = s_cnt[0];
        n_kv_t[1] = s_cnt[1];
    } else {
        n_kv_t[0] = p.causal ? min(tile[0] + 1, p.n_tiles_k) : p.n_tiles_k;
        n_kv_t[1] = has_b ? (p.causal ? min(tile[1] + 1, p.n_tiles_k) : p.n_tiles_k) : 0;
    }
    const int n_kv = sparse ? s_cnt[2] : (n_kv_t[0] > n_kv_t[1] ? n_kv_t[0] : n_kv_t[1]);
    const bool load_q[2] = {n_kv_t[0] > 0, n_kv_t[1] > 0};
    // The shared-memory list holds kMaxMaskTiles steps of 14-bit key tiles;
    // beyond that each thread walks the mask rows itself.
    const bool walk = sparse && (s_cnt[2] > kMaxMaskTiles || p.n_tiles_k > 0x4000);

    MaskWalk walker;
    auto kv_of = [&](int j) {
        if (!sparse) return j;
        return walk ? walker.at(j, p.n_tiles_k, [&](int x) { return s_pr.any(x); }) : static_cast<int>(s_kv[j] & 0x3FFF);
    };
    // Block-sparse: which query tiles take union step j (bit t for tile t).
    auto step_bits = [&](int j) -> unsigned {
        if (!walk) return (s_kv[j] >> 14) & 3u;
        const int kv = kv_of(j);
        return (s_pr.on(0, kv) ? 1u : 0u) | (s_pr.on(1, kv) ? 2u : 0u);
    };

    // Each warpgroup changes its register count inside its own branch, so the
    // compiler allocates each role's code for the count that role runs with.
    if (warp < 4) {
    ptx::setmaxnreg_dec<Cfg::kRegsLow>();
    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        // (no Q load for a query tile without key steps: its epilogue stages
        // zeros in that Q slot)
        if (lane == 0 && (!SPARSE || n_kv > 0)) {
            ptx::prefetch_tmap(&tm_q);
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            const uint64_t keep = ptx::policy_evict_last();
            ptx::mbar_arrive_expect_tx(&bar_q_full, ((load_q[0] ? 1 : 0) + (load_q[1] ? 1 : 0)) * G::kTileBytesK);
            for (int t = 0; t < 2; ++t) {
                if (!load_q[t]) continue;
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d(sQ[t] + b * kTileRows * G::kRowBK, &tm_q, &bar_q_full,
                                     b * G::kBoxK, tile[t] * kTileRows, bh);
            }
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % ST;
                const uint32_t ph = ((j / ST) & 1) ^ 1;
                if (j >= ST && !ptx::mbar_wait(&bar_k_empty[s], ph, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_k_full[s], G::kTileBytesK);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d_hint(sK + s * G::kTileBytesK + b * kTileRows * G::kRowBK, &tm_k,
                                          &bar_k_full[s], b * G::kBoxK, kv_of(j) * kTileRows, bh_kv, keep);
                k_issued = j + 1;
                if (j >= ST && !ptx::mbar_wait(&bar_v_empty[s], ph, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_v_full[s], G::kTileBytesMN);
                for (int b = 0; b < G::kNBoxMN; ++b)
                    ptx::tma_load_3d_hint(sV + s * G::kTileBytesMN + b * kTileRows * G::kRowBMN, &tm_v,
                                          &bar_v_full[s], b * G::kBoxMN, kv_of(j) * kTileRows, bh_kv, keep);
                v_issued = j + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                ptx::mbar_wait_drain(&bar_q_full, 0, kDrainNs);
                for (int t = k_issued - 1; t >= 0 && t >= k_issued - ST; --t)
                    ptx::mbar_wait_drain(&bar_k_full[t % ST], (t / ST) & 1, kDrainNs);
                for (int t = v_issued - 1; t >= 0 && t >= v_issued - ST; --t)
                    ptx::mbar_wait_drain(&bar_v_full[t % ST], (t / ST) & 1, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && (!SPARSE || n_kv > 0)) {
            constexpr uint32_t idesc_qk = ptx::instr_desc(G::kFmt, 128, 128, false, false);
            constexpr uint32_t idesc_pv = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            const uint32_t q_addr[2] = {ptx::smem_addr(sQ[0]), ptx::smem_addr(sQ[1])};
            bool ok = ptx::mbar_wait(q_go, 0, &abort_flag, tmo);
            auto issue_s = [&](int t, int j) {
                const uint32_t k_addr = ptx::smem_addr(sK + (j % ST) * G::kTileBytesK);
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk) {
                    const uint64_t a = desc_kmajor<G>(q_addr[t], kk);
                    const uint64_t b = desc_kmajor<G>(k_addr, kk);
                    if constexpr (G::kF32)
                        ptx::mma_tf32_ss(tmem + Cfg::col_s(t), a, b, idesc_qk, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_f16_ss(tmem + Cfg::col_s(t), a, b, idesc_qk, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bar_s_full[t]);
            };
            auto issue_pv = [&](int t, int j) -> bool {
                if (!ptx::mbar_wait(&bar_p_full[t], j & 1, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t v_addr = ptx::smem_addr(sV + (j % ST) * G::kTileBytesMN);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk) {
                    const uint64_t b = desc_mnmajor<G>(v_addr, kk);
                    const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
                    if constexpr (G::kF32)
                        ptx::mma_tf32_ts(tmem + Cfg::col_o(t), tmem + Cfg::col_s(t) + kk * 8, b, idesc_pv, acc);
                    else
                        ptx::mma_f16_ts(tmem + Cfg::col_o(t), tmem + Cfg::col_s(t) + kk * 8, b, idesc_pv, acc);
                }
                ptx::mma_commit(&bar_o_done[t]);
                return true;
            };
            if constexpr (SPARSE) {
                // Union step j: first the PV of each tile's previous step (step j-1,
                // still in the V ring), then S of the tiles whose block j is set; a
                // tile's PV always precedes its next S, which overwrites its P.  The
                // loads are checked here (a tile may skip steps, so no P barrier
                // covers them).
                int local[2] = {0, 0};         // steps issued per tile
                int pend[2] = {-1, -1};        // union step whose PV is still due
                auto flush = [&](int t) -> bool {
                    if (pend[t] < 0) return true;
                    const int l = local[t] - 1, jv = pend[t];
                    if (!ptx::mbar_wait(&bar_p_full[t], l & 1, &abort_flag, tmo)) return false;
                    if (!ptx::mbar_wait(&v_go[jv % ST], (jv / ST) & 1, &abort_flag, tmo)) return false;
                    ptx::tc_fence_after();
                    const uint32_t v_addr = ptx::smem_addr(sV + (jv % ST) * G::kTileBytesMN);
#pragma unroll
                    for (int kk = 0; kk < G::kStepsRows; ++kk) {
                        const uint64_t b = desc_mnmajor<G>(v_addr, kk);
                        const uint32_t acc = (l > 0 || kk > 0) ? 1u : 0u;
                        if constexpr (G::kF32)
                            ptx::mma_tf32_ts(tmem + Cfg::col_o(t), tmem + Cfg::col_s(t) + kk * 8, b, idesc_pv, acc);
                        else
                            ptx::mma_f16_ts(tmem + Cfg::col_o(t), tmem + Cfg::col_s(t) + kk * 8, b, idesc_pv, acc);
                    }
                    ptx::mma_commit(&bar_o_done[t]);
                    pend[t] = -1;
                    return true;
                };
                for (int j = 0; ok && j < n_kv; ++j) {
                    const unsigned bits = step_bits(j);
                    ok = ptx::mbar_wait(&k_go[j % ST], (j / ST) & 1, &abort_flag, tmo);
                    for (int t = 0; t < 2 && ok; ++t) {
                        if (!flush(t)) { ok = false; break; }
                        if ((bits >> t) & 1u) {
                            ptx::tc_fence_after();
                            issue_s(t, j);
                            pend[t] = j;
                            ++local[t];
                        }
                    }
                    if (!ok) break;
                    ptx::mma_commit(&bar_k_empty[j % ST]);
                    if (j > 0) ptx::mma_commit(&bar_v_empty[(j - 1) % ST]);
                }
                for (int t = 0; t < 2 && ok; ++t)
                    if (!flush(t)) ok = false;
                if (ok) ptx::mma_commit(&bar_v_empty[(n_kv - 1) % ST]);
            } else {
            // Prologue: S_A(0), S_B(0).
            if (ok) ok = ptx::mbar_wait(&k_go[0], 0, &abort_flag, tmo);
            if (ok) {
                ptx::tc_fence_after();
                issue_s(0, 0);
                if (n_kv_t[1] > 0) issue_s(1, 0);
                ptx::mma_commit(&bar_k_empty[0]);
            }
            // P_t(j) ready also means V_j and K_{j+1} have landed: the load watcher
            // (warp 2) checks them before its arrival on that barrier, so this
            // thread waits only on P (each wait here stalls it behind its own
            // pending MMAs).  Every key tile j < n_kv is used by the query tile
            // with the most steps, so both slots are released only after a
            // checked load.
            for (int j = 0; ok && j < n_kv; ++j) {
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j < n_kv_t[t]) {
                        if (!issue_pv(t, j)) { ok = false; break; }
                    }
                    if (j + 1 < n_kv_t[t]) issue_s(t, j + 1);
                }
                if (!ok) break;
                ptx::mma_commit(&bar_v_empty[j % ST]);
                if (j + 1 < n_kv) ptx::mma_commit(&bar_k_empty[(j + 1) % ST]);
            }
            }
            if (!ok) {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else if (warp == 2) {
        // ------------------------------------------------ load watcher
        // For step j of query tile t: once V_j and (if tile t goes on) K_{j+1}
        // have landed and the barrier's previous phase is complete, add the
        // fifth arrival to P_t(j)'s barrier, so that the issuer's wait on P
        // covers the loads too.  Off every critical path: it runs ahead of the
        // softmax groups by up to one phase.
        if (lane == 0 && !SPARSE) {
            bool ok = true;
            for (int j = 0; ok && j < n_kv; ++j) {
                for (int t = 0; t < 2 && ok; ++t) {
                    if (j >= n_kv_t[t]) continue;
                    ok = ptx::mbar_wait(&v_go[j % ST], (j / ST) & 1, &abort_flag, tmo);
                    if (ok && j + 1 < n_kv_t[t])
                        ok = ptx::mbar_wait(&k_go[(j + 1) % ST], ((j + 1) / ST) & 1, &abort_flag, tmo);
                    if (ok && j > 0) ok = ptx::mbar_wait(&bar_p_full[t], (j - 1) & 1, &abort_flag, tmo);
                    if (ok) ptx::mbar_arrive(&bar_p_full[t]);
                }
            }
        }
    } else if (G::kF32 && warp == 3) {
        // ------------------------------------------------ TF32 rounding (fp32 only)
        // Only the Q slots that were loaded: an unloaded slot stages the zero
        // epilogue of a query tile without key steps.
        if constexpr (G::kF32) {
            // Batched rounding loop at d = 64, the plain one at d <= 32 (as in the
            // one-tile kernel).
            constexpr bool kB = D >= 64;
            bool ok = (!SPARSE || n_kv > 0) && ptx::mbar_wait(&bar_q_full, 0, &abort_flag, tmo);
            if (ok) {
                for (int t = 0; t < 2; ++t)
                    if (load_q[t]) round_tf32_smem<G::kTileBytesK, kB>(sQ[t], lane);
                if (lane == 0) ptx::mbar_arrive(&bar_q_ready);
            }
            for (int j = 0; ok && j < n_kv; ++j) {
                const int s = j % ST;
                if (!ptx::mbar_wait(&bar_k_full[s], (j / ST) & 1, &abort_flag, tmo)) break;
                round_tf32_smem<G::kTileBytesK, kB>(sK + s * G::kTileBytesK, lane);
                if (lane == 0) ptx::mbar_arrive(&bar_k_ready[s]);
                if (!ptx::mbar_wait(&bar_v_full[s], (j / ST) & 1, &abort_flag, tmo)) break;
                round_tf32_smem<G::kTileBytesMN, kB>(sV + s * G::kTileBytesMN, lane);
                if (lane == 0) ptx::mbar_arrive(&bar_v_ready[s]);
            }
        }
    }
    } else {
        ptx::setmaxnreg_inc<Cfg::kRegsHigh>();
        // ------------------------------------------------ softmax warpgroups
        const int t = (warp - 4) >> 2;       // 0: warps 4-7 (tile A), 1: warps 8-11 (tile B)
        // Every existing query tile writes O and L, also one without key steps.
        if (SPARSE ? tile[t] < p.n_tiles : n_kv_t[t] > 0) {
            fwd2_softmax<ES, D, F16, SPARSE>(p, t, tile[t], n_kv_t[t], bh, tmem, sQ[t], &bar_s_full[t],
                                &bar_p_full[t], &bar_o_done[t], &s_pr, &abort_flag, &tm_o);
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
