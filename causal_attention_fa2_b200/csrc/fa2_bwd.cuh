// fa2_bwd.cuh -- FlashAttention-2 backward pass with recomputation for sm_100a.
//
// The handout's backward (CS336 A2 Systems handout section 4.2.2, "backward
// pass with recomputation", Eqs. 13-19):
//   D   = rowsum(O o dO)                       (computed once, before the loop)
//   S   = scale Q K^T,  P_ij = exp(S_ij - L_i)  (Eqs. 13-14, recomputed)
//   dV  = P^T dO,  dP = dO V^T                 (Eqs. 15-16)
//   dS_ij = P_ij (dP_ij - D_i)                 (Eq. 17)
//   dQ  = scale dS K,  dK = scale dS^T Q        (Eqs. 18-19)
// organised as the handout's tiled Algorithm 2 (section 4.2.3) describes it:
// P is computed twice, once in a pass that owns a key/value tile and
// accumulates its dK and dV, once in a pass that owns a query tile and
// accumulates its dQ, so no partial result is ever added across thread
// blocks (no atomics, and every output is deterministic).
//
// Three kernels, enqueued back to back on one stream:
//   fa2_bwd_pre_kernel    per query row: D_i and L_i * log2(e), padded to
//                         whole 128-row tiles with 0 / +inf so padded rows
//                         drop out of P and dS.
//   fa2_bwd_dkdv_kernel   one CTA per (key tile j, key/value head), looping over
//                         the (query head, query tile i) steps that see key
//                         tile j (i >= j causal); with grouped-query heads and
//                         few key tiles the steps are split over several CTAs
//                         whose fp32 partials fa2_bwd_kv_reduce_kernel sums.
//   fa2_bwd_dq_kernel     one CTA per (query tile i, head), looping over the
//                         key tiles j that query tile i sees (j <= i causal).
//
// Both main kernels use warp 0 as TMA producer, warp 1 as MMA issuer (one
// thread) and warps 2-5 and 6-9 as two elementwise groups; the dQ pass adds
// warp 10 as a second MMA issuer.  The thread holding TMEM lane t of either
// group owns row t of the 128-row tile the CTA owns; group g handles columns
// [64g, 64g+64) of the 128 x 128 score tile.  P and dS are written back into
// tensor memory over the scores they came from (bf16 pairs) and read by the
// next MMA as its A operand, so the elementwise groups never write shared
// memory on the hot path.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "fa2_traits.cuh"

namespace fa2 {

// Workspace carved out of the caller's buffer (every region 256-byte aligned):
// L*log2(e) and D, fp32, [BH][n_pad]; for 4-byte inputs also copies of q and
// dout ([BH][N][d]) and of k and v ([BH_kv][Nk][d]) rounded to TF32 (offsets 0
// when absent).
struct BwdWorkspace {
    size_t l2_off, d_off, q_off, k_off, v_off, do_off, part_off, dqacc_off, total;
    int n_pad;
    int kv_splits;   // dK/dV pass: CTAs per (key tile, key/value head)
};

inline size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// With few key/value heads (grouped-query / multi-query attention) the dK/dV
// pass has few CTAs: n_tiles_k * BH_kv of them, each looping over its whole
// query-head group.  Below kSplitMinCtas CTAs the (query head, query tile)
// steps of a group are split over up to `group` CTAs, each writing fp32 partial
// dK, dV that a reduction pass sums in split order (so results stay
// deterministic).  A function of the shapes only, so the workspace size does
// not depend on the device.
constexpr int kSplitMinCtas = 148;
constexpr int kSplitTargetCtas = 296;
__host__ __device__ inline int dkdv_splits(int n_tiles_k, int BH_kv, int group) {
    const long long ctas = static_cast<long long>(n_tiles_k) * BH_kv;
    if (group <= 1 || ctas >= kSplitMinCtas) return 1;
    const long long want = (kSplitTargetCtas + ctas - 1) / ctas;
    return static_cast<int>(want < group ? want : group);
}

// The one-pass backward (fa2_bwd_fused.cuh) runs where it applies: 16-bit
// inputs, no block mask, no split dK/dV groups, more than one key tile.
inline bool one_pass_applies(int n_tiles_k, int elem_bytes, int kv_splits, bool block_sparse) {
    return elem_bytes == 2 && !block_sparse && kv_splits == 1 && n_tiles_k > 1;
}

// with_dq_acc: also reserve the one-pass backward's fp32 dQ accumulator
// [BH][n_pad][d] when the one-pass backward applies to these sizes.
inline BwdWorkspace bwd_workspace_layout(int BH, int N, int BH_kv, int Nk, int d, int elem_bytes,
                                         bool with_dq_acc = true) {
    BwdWorkspace w;
    w.n_pad = (N + kTileRows - 1) / kTileRows * kTileRows;
    const size_t vec = align256(static_cast<size_t>(BH) * w.n_pad * sizeof(float));
    w.l2_off = 0;
    w.d_off = vec;
    w.total = 2 * vec;
    w.q_off = w.k_off = w.v_off = w.do_off = w.part_off = w.dqacc_off = 0;
    const int n_tiles_k = (Nk + kTileRows - 1) / kTileRows;
    w.kv_splits = elem_bytes == 2 ? dkdv_splits(n_tiles_k, BH_kv, BH / BH_kv) : 1;
    if (w.kv_splits > 1) {
        // fp32 partial dK and dV: [2][splits][BH_kv][n_tiles_k * 128][d]
        w.part_off = w.total;
        w.total += align256(2ull * w.kv_splits * BH_kv * n_tiles_k * kTileRows * d * sizeof(float));
    }
    if (with_dq_acc && one_pass_applies(n_tiles_k, elem_bytes, w.kv_splits, false)) {
        w.dqacc_off = w.total;
        w.total += align256(static_cast<size_t>(BH) * w.n_pad * d * sizeof(float));
    }
    if (elem_bytes == 4) {
        const size_t tq = align256(static_cast<size_t>(BH) * N * d * sizeof(float));
        const size_t tk = align256(static_cast<size_t>(BH_kv) * Nk * d * sizeof(float));
        w.q_off = w.total;
        w.k_off = w.q_off + tq;
        w.v_off = w.k_off + tk;
        w.do_off = w.v_off + tk;
        w.total = w.do_off + tq;
    }
    return w;
}

// ------------------------------------------------------------------ pre-processing

// Geometry of the pre-pass: a row of d 16-bit values is read as 16-byte
// vectors, kPer of them per thread, by kTPR threads (rounded up to a power of
// two), so one warp covers 32 / kTPR rows and one 256-thread block 8 * 32 / kTPR
// rows.
template <int D>
struct BwdPreCfg {
    static constexpr int kVec = 8;                                  // elements per 16-byte load
    static constexpr int kChunks = (D + kVec - 1) / kVec;          // 16-byte chunks per row
    // Two chunks of O and of dO per thread from d = 64 up, so four 16-byte loads
    // are in flight per thread.
    static constexpr int kPer = kChunks >= 8 ? 2 : 1;
    static constexpr int kUsed = (kChunks + kPer - 1) / kPer;      // threads that load
    static constexpr int kTPR = kUsed <= 2 ? 2 : kUsed <= 4 ? 4 : kUsed <= 8 ? 8 : 16;
    static constexpr int kRowsPerBlock = 8 * 32 / kTPR;
};

// D_i = rowsum(O_i o dO_i) and L_i * log2(e) per query row; rows past N (up
// to the padded length) get D = 0 and L = +inf so they drop out of P and dS.
// O and dO are 16-bit (bf16, or fp16 when F16), read as raw 16-bit pairs.
// With dq_acc (the one-pass backward's fp32 dQ accumulator, [BH][n_pad][D])
// the row is also zeroed there.
template <int D, bool F16 = false>
__global__ void __launch_bounds__(256)
fa2_bwd_pre_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout,
                   const float* __restrict__ lse, float* __restrict__ l2,
                   float* __restrict__ dvec, int N, int n_pad, long long rows_total,
                   float* __restrict__ dq_acc = nullptr) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using C = BwdPreCfg<D>;
    const int sub = threadIdx.x % C::kTPR;
    const long long row = static_cast<long long>(blockIdx.x) * C::kRowsPerBlock + threadIdx.x / C::kTPR;
    const bool live = row < rows_total;
    const long long bh = row / n_pad;
    const int n = static_cast<int>(row - bh * n_pad);
    float acc = 0.f;
    if (dq_acc && live && sub < C::kUsed) {
#pragma unroll
        for (int e = 0; e < C::kPer; ++e) {
            float4* z = reinterpret_cast<float4*>(dq_acc + row * D + (sub * C::kPer + e) * C::kVec);
            z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
            z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    if (live && n < N && sub < C::kUsed) {
        const size_t base = (static_cast<size_t>(bh) * N + n) * D + sub * C::kPer * C::kVec;
        uint4 a[C::kPer], b[C::kPer];
#pragma unroll
        for (int e = 0; e < C::kPer; ++e) {
            a[e] = __ldg(reinterpret_cast<const uint4*>(o + base) + e);
            b[e] = __ldg(reinterpret_cast<const uint4*>(dout + base) + e);
        }
#pragma unroll
        for (int e = 0; e < C::kPer; ++e) {
            const uint32_t aw[4] = {a[e].x, a[e].y, a[e].z, a[e].w};
            const uint32_t bw[4] = {b[e].x, b[e].y, b[e].z, b[e].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                float a0, a1, b0, b1;
                TileGeom<2, D, F16>::unpack2(aw[w], a0, a1);
                TileGeom<2, D, F16>::unpack2(bw[w], b0, b1);
                acc = fmaf(a0, b0, acc);
                acc = fmaf(a1, b1, acc);
            }
        }
    }
#pragma unroll
    for (int off = C::kTPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (live && sub == 0) {
        if (n < N) {
            dvec[row] = acc;
            l2[row] = lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f;
        } else {
            dvec[row] = 0.f;
            l2[row] = INFINITY;
        }
    }
}

// ------------------------------------------------------------------ shared pieces

struct BwdParams {
    const float* l2;       // [BH][n_pad]  L * log2(e), +inf past N
    float* dvec;           // [BH][n_pad]  D, 0 past N (the dQ pass rewrites the
                           // rows of a query tile that sees a single key tile)
    uint32_t* status;
    int N, BH, n_tiles, n_pad, causal;   // query length, B * H, query tiles, padded rows
    int Nk, n_tiles_k;                   // key/value length and tiles
    int H, H_kv, group, BH_kv;   // query heads, key/value heads, H / H_kv, B * H_kv
    float scale_log2;      // scale * log2(e)
    float scale;
    unsigned long long timeout_ns;
    const uint8_t* block_mask;  // [n_tiles][n_tiles_k] block mask, or nullptr (dense)
    int kv_splits;         // dK/dV pass CTAs per (key tile, key/value head)
    float* part;           // fp32 partial dK, dV when kv_splits > 1
    int item0;             // dQ pass: work item of the first CTA (a launch may cover a suffix)
    int head_group;        // heads (dK/dV pass: key/value heads x splits) per group of work items
    const float* k32;      // fp32 dK/dV pass at d = 128: TF32-rounded K, [BH_kv][Nk][D]
    const float* q32;      // fp32 dQ pass at d = 128: TF32-rounded Q and dO, [BH][N][D]
    const float* do32;
};

template <int ES, int D, bool F16 = false>
struct BwdCfg {
    using G = TileGeom<ES, D, F16>;
    static_assert(ES == 2, "the backward kernels are written for 16-bit inputs");
    // Warp 0 TMA producer, warp 1 MMA issuer, warps 2-9 the two elementwise
    // groups; the dQ pass adds warp 10 as a second MMA issuer.
    static constexpr int kThreads = 320;
    static constexpr int kThreadsDq = 352;
    static constexpr int kTile = G::kTileBytesK;
    // 227 KB minus the alignment pad and the static shared memory.
    static constexpr int kBudget = 227 * 1024 - 1024 - 10 * 1024;
    // Two resident tiles (K,V or Q,dO) plus two rings of streamed tiles.
    static constexpr int kRing0 = (kBudget - 2 * kTile) / (2 * kTile);
    static constexpr int kRing = kRing0 > 3 ? 3 : kRing0;
    static_assert(kRing >= 2, "shared memory too small for the streaming rings");
    static constexpr int kSmemBytes = 1024 + 2 * kTile + 2 * kRing * kTile;
    // dQ pass (static shared memory under 2 KB): Q, dO resident, K and V
    // streamed.  K_j stays until dQ += dS K_j has read it, two MMA groups
    // after S(j), so K takes the deeper ring.
    static constexpr int kDqStream = (227 * 1024 - 1024 - 2048) / kTile - 2;
    static constexpr int kRingK = kDqStream - 2 > 3 ? 3 : kDqStream - 2;
    static constexpr int kRingV = kDqStream - kRingK > 3 ? 3 : kDqStream - kRingK;
    static_assert(kRingK >= 2 && kRingV >= 2, "shared memory too small for the dQ rings");
    static constexpr int kDqSmemBytes = 1024 + (2 + kRingK + kRingV) * kTile;
    static constexpr uint32_t kTmemCols = 512;
    // dK/dV pass: S^T | dP^T | dV | dK.   dQ pass: S | dP (even key tiles) | dQ |
    // dP (odd key tiles); dQ takes at most 128 columns.
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384, kColDQ = 256;
    static constexpr uint32_t kColDP1 = 384;
    static_assert(G::kNOut <= 128, "dQ must fit between the two dP buffers");
};

// TMEM column, relative to the score (or dP) block, of k-step kk of the
// 16-bit P (or dS) A operand.  The group that owns columns [64g, 64g + 64)
// writes its 64 values, packed two per column, to the first 32 of them, so
// k-steps 4g .. 4g+3 read there and neither group waits for the other.
__host__ __device__ constexpr uint32_t a_col(int kk) {
    return static_cast<uint32_t>((kk / 4) * 64 + (kk % 4) * 8);
}

// ------------------------------------------------------------------ dK / dV pass

// Per query tile i the MMA issuer runs
//   dV += P^T(i) dO(i)      (A = P^T from TMEM)     ; S^T(i+1) = K Q(i+1)^T
//   dK += dS^T(i) Q(i)      (A = dS^T from TMEM)    ; dP^T(i+1) = V dO(i+1)^T
// while the groups compute P^T(i+1) and dS^T(i+1).
template <int ES, int D, bool F16 = false, bool SPARSE = false>
__global__ void __launch_bounds__(320, 1)
fa2_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                    const BwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = BwdCfg<ES, D, F16>;
    using G = typename Cfg::G;
    constexpr int RS = Cfg::kRing;
    constexpr int TB = Cfg::kTile;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kv_full;
    __shared__ uint64_t bar_q_full[RS], bar_q_empty[RS], bar_do_full[RS], bar_do_empty[RS];
    __shared__ uint64_t bar_s_full, bar_dp_full, bar_p_ready, bar_ds_ready;
    __shared__ uint64_t bar_dkv_full, bar_drain;
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    // Per-warp copies of the current query tile's L*log2(e) and D values for
    // the warp's 64 query columns (double-buffered; each warp syncs itself).
    __shared__ __align__(16) float sL2[8][2][64];
    __shared__ __align__(16) float sDv[8][2][64];
    // Block-sparse: the query tiles whose block with this key tile is set.
    __shared__ uint16_t s_q[SPARSE ? kMaxMaskTiles : 1];
    __shared__ int s_nq;
    // Block-sparse, causal: the query tile kv_tile (the diagonal step) has no set
    // block before this key tile, so its rows see this key tile only.
    __shared__ int s_diag_single;

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sK = smem;
    uint8_t* sV = sK + TB;
    uint8_t* sQr = sV + TB;
    uint8_t* sDOr = sQr + RS * TB;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: (key tile j, key/value head).  Key tile j is seen by query
    // tiles j..T-1 (causal) of each of the `group` query heads sharing this
    // key/value head, whose dK and dV sum over all of them; small j carries
    // the most work and is issued first.
    int kv_tile, item_r;
    grouped_item(blockIdx.x, p.n_tiles_k, p.BH_kv * p.kv_splits, p.head_group, kv_tile, item_r);
    const int split = item_r / p.BH_kv;                 // which share of the group's steps
    const int bh = item_r - split * p.BH_kv;            // key/value head
    const int i_begin = p.causal ? kv_tile : 0;
    const int kv_row0 = kv_tile * kTileRows;
    constexpr bool sparse = SPARSE;
    const int n_col = p.n_tiles > i_begin ? p.n_tiles - i_begin : 0;   // candidate query tiles
    auto blk_set = [&](int t) { return __ldg(p.block_mask + static_cast<size_t>(i_begin + t) * p.n_tiles_k + kv_tile) != 0; };
    if (sparse && warp == 0) {
        const int n = warp_compact(s_q, n_col, blk_set, [&](int t) { return i_begin + t; });
        bool before = false;
        if (p.causal && kv_tile < p.n_tiles) {
            const uint8_t* row = p.block_mask + static_cast<size_t>(kv_tile) * p.n_tiles_k;
            for (int base = 0; base < kv_tile; base += 32)
                before |= __any_sync(0xffffffffu, base + lane < kv_tile && row[base + lane] != 0);
        }
        if (lane == 0) { s_nq = n; s_diag_single = before ? 0 : 1; }
    }

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
    // Query tiles per query head; none when no query reaches this key tile
    // (causal with keys longer than queries, or an empty block column): then
    // dK = dV = 0 is written.
    const int n_q = sparse ? s_nq : n_col;
    // Past kMaxMaskTiles steps (or 16-bit tile indices) each thread walks the column.
    const bool walk = sparse && (n_q > kMaxMaskTiles || p.n_tiles > 0xFFFF);
    MaskWalk walker;
    // (query head, query tile) steps of the group, this CTA taking the split-th
    // of kv_splits consecutive shares.
    const int n_all = n_q * p.group;
    const int share = (n_all + p.kv_splits - 1) / p.kv_splits;
    const int it0 = min(split * share, n_all);
    const int n_it = min(n_all - it0, share);
    // Step it: global step it0 + it = (query head) * n_q + (query tile index).
    auto q_tile_of = [&](int it) {
        const int g = (it0 + it) % n_q;
        if (!sparse) return i_begin + g;
        return walk ? i_begin + walker.at(g, n_col, blk_set) : static_cast<int>(s_q[g]);
    };
    auto q_head_of = [&](int it) { return (bh / p.H_kv) * p.H + (bh % p.H_kv) * p.group + (it0 + it) / n_q; };
    // Steps whose query tile sees this key tile only (causal: query tile 0, or
    // with a block mask the diagonal step of a block row with nothing before
    // it; or a single key tile), where rows see few keys and |dS| is of the
    // order of |dP|: dS^T goes to the dK MMA as two 16-bit parts hi + lo, so it
    // is not rounded before the contraction.  With a mask of all ones this is
    // the rule without a mask.
    auto hilo_of = [&](int i) {
        return p.n_tiles_k == 1 || (p.causal && (sparse ? (i == kv_tile && s_diag_single != 0) : i == 0));
    };

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
            const uint32_t k_addr = ptx::smem_addr(sK);
            const uint32_t v_addr = ptx::smem_addr(sV);
            auto q_addr = [&](int it) { return ptx::smem_addr(sQr + (it % RS) * TB); };
            auto do_addr = [&](int it) { return ptx::smem_addr(sDOr + (it % RS) * TB); };
            // S^T = K_j Q_i^T   (Eq. 13, transposed: rows are keys)
            // Q_i / dO_i of step i >= 1 have landed once the groups report P^T / dS^T
            // of step i-1 (one thread checks them before arriving), so only step 0
            // waits on the loads here: each such wait stalls this thread behind its
            // pending MMAs.
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
            // dP^T = V_j dO_i^T   (Eq. 16, transposed)
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
            bool ok = ptx::mbar_wait(&bar_kv_full, 0, &abort_flag, tmo);
            if (ok) ok = issue_s(0) && issue_dp(0);
            for (int it = 0; ok && it < n_it; ++it) {
                // dV_j += P^T dO_i   (Eq. 15); P^T read from the score columns.
                if (!ptx::mbar_wait(&bar_p_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t da = do_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ts(tmem + Cfg::kColDV, tmem + Cfg::kColS + a_col(kk), desc_mnmajor<G>(da, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar_do_empty[it % RS]);
                if (it + 1 < n_it && !issue_s(it + 1)) { ok = false; break; }
                // dK_j += dS^T Q_i   (Eq. 19 without the scale); dS^T from the dP^T columns.
                if (!ptx::mbar_wait(&bar_ds_ready, it & 1, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t qa = q_addr(it);
#pragma unroll
                for (int kk = 0; kk < G::kStepsRows; ++kk)
                    ptx::mma_f16_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDP + a_col(kk), desc_mnmajor<G>(qa, kk), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                if (hilo_of(q_tile_of(it))) {
                    // dK_j += dS^T_lo Q_i: the low parts sit 32 columns after the high parts.
#pragma unroll
                    for (int kk = 0; kk < G::kStepsRows; ++kk)
                        ptx::mma_f16_ts(tmem + Cfg::kColDK, tmem + Cfg::kColDP + a_col(kk) + 32, desc_mnmajor<G>(qa, kk), idesc_kv, 1u);
                }
                ptx::mma_commit(&bar_q_empty[it % RS]);
                if (it + 1 < n_it && !issue_dp(it + 1)) { ok = false; break; }
            }
            if (ok) {
                ptx::mma_commit(&bar_dkv_full);
            } else {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else {
        // ------------------------------------------------ two P / dS groups
        const int g = (warp - 2) >> 2;                  // query columns [64g, 64g+64)
        const int wi = warp - 2;
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // key row inside the tile
        const int qc0 = 64 * g;
        const bool key_valid = kv_row0 + r < p.Nk;
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        // Offset of step it's L / D values for this group's 64 query columns.
        auto vec_base = [&](int it) {
            return static_cast<size_t>(q_head_of(it)) * p.n_pad + static_cast<size_t>(q_tile_of(it)) * kTileRows + qc0;
        };
        float nl2[2] = {0.f, 0.f}, nd[2] = {0.f, 0.f};
        if (n_it > 0) {
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                nl2[m] = p.l2[vec_base(0) + lane + 32 * m];
                nd[m] = p.dvec[vec_base(0) + lane + 32 * m];
            }
        }
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
            const int i = q_tile_of(it);
            const int b = it & 1;
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                sL2[wi][b][lane + 32 * m] = nl2[m];
                sDv[wi][b][lane + 32 * m] = nd[m];
            }
            __syncwarp();
            if (it + 1 < n_it) {
                const size_t nb = vec_base(it + 1);
#pragma unroll
                for (int m = 0; m < 2; ++m) {
                    nl2[m] = p.l2[nb + lane + 32 * m];
                    nd[m] = p.dvec[nb + lane + 32 * m];
                }
            }
            const bool diag = p.causal && (i == kv_tile);
            // ---- P^T = exp2(S^T * scale*log2(e) - L*log2(e))   (Eq. 14)
            if (!ptx::mbar_wait(&bar_s_full, it & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pk[32];                               // this group's P^T row, bf16 pairs
            {
                uint32_t us[64];
                ptx::tmem_ld32(lane_base + Cfg::kColS + qc0, *reinterpret_cast<uint32_t(*)[32]>(us));
                ptx::tmem_ld32(lane_base + Cfg::kColS + qc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(us + 32));
                ptx::tmem_wait_ld();
                const float2 sl2v = make_float2(sl2, sl2);
                if (diag || !key_valid) {
#pragma unroll
                    for (int c = 0; c < 64; c += 4) {
                        const float4 lv = *reinterpret_cast<const float4*>(&sL2[wi][b][c]);
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
                        const float4 lv = *reinterpret_cast<const float4*>(&sL2[wi][b][c]);
                        const float2 a0 = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, make_float2(-lv.x, -lv.y));
                        const float2 a1 = ptx::fma2(make_float2(__uint_as_float(us[c + 2]), __uint_as_float(us[c + 3])), sl2v, make_float2(-lv.z, -lv.w));
                        pk[c >> 1] = G::pack2(ptx::ex2_approx(a0.x), ptx::ex2_approx(a0.y));
                        pk[(c >> 1) + 1] = G::pack2(ptx::ex2_approx(a1.x), ptx::ex2_approx(a1.y));
                    }
                }
            }
            // P^T -> this group's own score columns [64g, 64g + 32) (already read,
            // so no wait on the other group), A operand of dV += P^T dO.
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
            if (hilo_of(i)) {
                // dS^T = hi + lo, both rounded to the 16-bit type: hi into the group's
                // first 32 dP^T columns, lo into the next 32 (the issuer's second dK
                // group reads them).  Columns are overwritten only after they are read.
                uint32_t lo_a[16];
                {
                    uint32_t ud[32], hi[16];
                    ptx::tmem_ld32(lane_base + Cfg::kColDP + qc0, ud);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        float2 pp, hv;
                        G::unpack2(pk[c >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c]), __uint_as_float(ud[c + 1])),
                                                                  make_float2(-sDv[wi][b][c], -sDv[wi][b][c + 1])));
                        hi[c >> 1] = G::pack2(ds.x, ds.y);
                        G::unpack2(hi[c >> 1], hv.x, hv.y);
                        lo_a[c >> 1] = G::pack2(ds.x - hv.x, ds.y - hv.y);
                    }
                    ptx::tmem_st16(lane_base + Cfg::kColDP + qc0, hi);          // hi, values 0..31
                }
                {
                    uint32_t ud[32], hi[16], lo[16];
                    ptx::tmem_ld32(lane_base + Cfg::kColDP + qc0 + 32, ud);
                    ptx::tmem_wait_ld();
                    ptx::tmem_st16(lane_base + Cfg::kColDP + qc0 + 32, lo_a);     // lo, values 0..31
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        float2 pp, hv;
                        G::unpack2(pk[(32 + c) >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c]), __uint_as_float(ud[c + 1])),
                                                                  make_float2(-sDv[wi][b][32 + c], -sDv[wi][b][33 + c])));
                        hi[c >> 1] = G::pack2(ds.x, ds.y);
                        G::unpack2(hi[c >> 1], hv.x, hv.y);
                        lo[c >> 1] = G::pack2(ds.x - hv.x, ds.y - hv.y);
                    }
                    ptx::tmem_st16(lane_base + Cfg::kColDP + qc0 + 16, hi);     // hi, values 32..63
                    ptx::tmem_st16(lane_base + Cfg::kColDP + qc0 + 48, lo);     // lo, values 32..63
                }
            } else {
            uint32_t dk[32];                               // this group's dS^T row, bf16 pairs
            {
                uint32_t ud[64];
                ptx::tmem_ld32(lane_base + Cfg::kColDP + qc0, *reinterpret_cast<uint32_t(*)[32]>(ud));
                ptx::tmem_ld32(lane_base + Cfg::kColDP + qc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(ud + 32));
                ptx::tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 64; c += 4) {
                    const float4 dv4 = *reinterpret_cast<const float4*>(&sDv[wi][b][c]);
                    const float2 nd[2] = {make_float2(-dv4.x, -dv4.y), make_float2(-dv4.z, -dv4.w)};
#pragma unroll
                    for (int h = 0; h < 4; h += 2) {
                        float2 pp;
                        G::unpack2(pk[(c + h) >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c + h]), __uint_as_float(ud[c + h + 1])), nd[h >> 1]));
                        dk[(c + h) >> 1] = G::pack2(ds.x, ds.y);
                    }
                }
            }
            // dS^T -> this group's own dP^T columns [128 + 64g, ... + 32), A operand
            // of dK += dS^T Q.
            ptx::tmem_st32(lane_base + Cfg::kColDP + qc0, dk);
            }
            ptx::tmem_wait_st();
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
        if (p.kv_splits > 1) {
            // Split group: this CTA's fp32 partial sums, one key row per thread, to
            // part[dK = 0 / dV = 1][split][head][row][d]; the reduction pass scales
            // dK, sums the splits in order and rounds.
            if (ok) {
                ptx::tc_fence_after();
                const uint32_t col = g == 0 ? Cfg::kColDV : Cfg::kColDK;
                const size_t nk_pad = static_cast<size_t>(p.n_tiles_k) * kTileRows;
                float* rowp = p.part + ((((g == 0 ? 1 : 0) * static_cast<size_t>(p.kv_splits) + split) *
                                         p.BH_kv + bh) * nk_pad + kv_row0 + r) * D;
#pragma unroll
                for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                    uint32_t u[16] = {};
                    if (n_it > 0) {
                        ptx::tmem_ld16(lane_base + col + c0, u);
                        ptx::tmem_wait_ld();
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        if (c0 + 4 * q4 < D)
                            *reinterpret_cast<float4*>(rowp + c0 + 4 * q4) =
                                make_float4(__uint_as_float(u[4 * q4]), __uint_as_float(u[4 * q4 + 1]),
                                            __uint_as_float(u[4 * q4 + 2]), __uint_as_float(u[4 * q4 + 3]));
                    }
                }
            }
        } else {
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

// dK, dV of a split group: element e of head hd, key row row (of Nk), column
// col = sum over the kv_splits partials in split order; dK times scale; rounded
// once to the 16-bit output type.  One thread per 4 consecutive columns.
template <bool F16>
__global__ void __launch_bounds__(256)
fa2_bwd_kv_reduce_kernel(const float* __restrict__ part, uint16_t* __restrict__ dk,
                         uint16_t* __restrict__ dv, int splits, int BH_kv, int Nk, int nk_pad, int d,
                         float scale) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    const size_t per = static_cast<size_t>(BH_kv) * Nk * d / 4;   // 4-column groups per tensor
    const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i >= 2 * per) return;
    const int which = i >= per ? 1 : 0;                              // 0: dK, 1: dV
    const size_t e = (i - which * per) * 4;
    const size_t hd = e / (static_cast<size_t>(Nk) * d);
    const size_t rem = e - hd * Nk * d;
    const size_t row = rem / d, col = rem - row * d;
    const size_t stride = static_cast<size_t>(BH_kv) * nk_pad * d;  // one split's tensor
    const float* src = part + (static_cast<size_t>(which) * splits * BH_kv + hd) * nk_pad * d + row * d + col;
    float4 acc = *reinterpret_cast<const float4*>(src);
    for (int s = 1; s < splits; ++s) {
        const float4 x = *reinterpret_cast<const float4*>(src + s * stride);
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
    }
    const float m = which == 0 ? scale : 1.f;
    uint2 w;
    if constexpr (F16) {
        w.x = ptx::pack_f16x2(acc.x * m, acc.y * m);
        w.y = ptx::pack_f16x2(acc.z * m, acc.w * m);
    } else {
        w.x = ptx::pack_bf16x2(acc.x * m, acc.y * m);
        w.y = ptx::pack_bf16x2(acc.z * m, acc.w * m);
    }
    *reinterpret_cast<uint2*>((which == 0 ? dk : dv) + e) = w;
}

// ------------------------------------------------------------------ dQ pass

// One CTA per (query tile i, head).  Per key tile j the tensor core runs
//   S(j) = Q K_j^T ; dP(j) = dO V_j^T ; dQ += dS(j) K_j   (A = dS from TMEM)
// from two issuing threads: S(j+1) as soon as both groups have read S(j), and
// dP into two TMEM buffers, dP(j+2) right after dQ(j) (which reads dS(j) from
// the same buffer), so dP(j+1) is ready when the groups finish P(j+1).  A
// thread that waits on an mbarrier after committing MMAs stalls until those
// MMAs are done; with two issuers the other one's MMAs keep the tensor core
// busy meanwhile.
template <int ES, int D, bool F16 = false, bool SPARSE = false>
__global__ void __launch_bounds__(352, 1)
fa2_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = BwdCfg<ES, D, F16>;
    using G = typename Cfg::G;
    constexpr int RK = Cfg::kRingK;
    constexpr int RV = Cfg::kRingV;
    constexpr int TB = Cfg::kTile;

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_qdo_full;
    __shared__ uint64_t bar_k_full[RK], bar_k_empty[RK], bar_v_full[RV], bar_v_empty[RV];
    // dP and dS of key tile j live in buffer j % 2, and so do their barriers: with
    // dP(j+1) issued before dQ(j) a warp may finish dS(j+1) while another still
    // works on dS(j), so one dS barrier would mix their arrivals.  (No warp gets
    // two key tiles ahead: S(j+2) is issued only after every warp read S(j+1).)
    __shared__ uint64_t bar_s_full, bar_dp_full[2], bar_s_read, bar_ds_ready[2];
    __shared__ uint64_t bar_dq_done, bar_drain[2];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    // Block-sparse: the key tiles whose block with this query tile is set.
    __shared__ uint16_t s_kv[SPARSE ? kMaxMaskTiles : 1];
    __shared__ int s_nkv;

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* sQ = smem;
    uint8_t* sDO = sQ + TB;
    uint8_t* sKr = sDO + TB;
    uint8_t* sVr = sKr + RK * TB;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: causal query tile i sees key tiles 0..i; longest first.  A
    // launch may cover only the last items (item0 > 0: the single-tile query
    // tiles ahead of the one-pass backward).
    int rank, bh;
    grouped_item(blockIdx.x + p.item0, p.n_tiles, p.BH, p.head_group, rank, bh);
    const int q_tile = p.causal ? (p.n_tiles - 1 - rank) : rank;
    // Key tiles this query tile sees (causal: key index <= query index).
    const int n_kv_lim = p.causal ? min(q_tile + 1, p.n_tiles_k) : p.n_tiles_k;
    constexpr bool sparse = SPARSE;
    const uint8_t* mask_row = sparse ? p.block_mask + static_cast<size_t>(q_tile) * p.n_tiles_k : nullptr;
    auto blk_set = [&](int j) { return __ldg(mask_row + j) != 0; };
    if (sparse && warp == 0) {
        const int n = warp_compact(s_kv, n_kv_lim, blk_set, [&](int j) { return j; });
        if (lane == 0) s_nkv = n;
    }
    const int q_row0 = q_tile * kTileRows;
    const int bh_kv = kv_head_of(bh, p.H, p.H_kv, p.group);

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_qdo_full, 1);
        for (int s = 0; s < RK; ++s) {
            ptx::mbar_init(&bar_k_full[s], 1);
            ptx::mbar_init(&bar_k_empty[s], 2);         // released by S(j) and dQ(j)
        }
        for (int s = 0; s < RV; ++s) {
            ptx::mbar_init(&bar_v_full[s], 1);
            ptx::mbar_init(&bar_v_empty[s], 1);
        }
        ptx::mbar_init(&bar_s_full, 1);
        ptx::mbar_init(&bar_dp_full[0], 1);
        ptx::mbar_init(&bar_dp_full[1], 1);
        ptx::mbar_init(&bar_s_read, 8);
        ptx::mbar_init(&bar_ds_ready[0], 8);
        ptx::mbar_init(&bar_ds_ready[1], 8);
        ptx::mbar_init(&bar_dq_done, 1);
        ptx::mbar_init(&bar_drain[0], 1);
        ptx::mbar_init(&bar_drain[1], 1);
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
    // Key-tile steps; none for an empty block row, whose dQ is written as 0
    // (nothing is loaded, so the Q slot can stage the zeros).
    const int n_kv = sparse ? s_nkv : n_kv_lim;
    // Past kMaxMaskTiles steps (or 16-bit tile indices) each thread walks the row.
    const bool walk = sparse && (n_kv > kMaxMaskTiles || p.n_tiles_k > 0xFFFF);
    MaskWalk walker;
    auto kv_of = [&](int j) {
        if (!sparse) return j;
        return walk ? walker.at(j, n_kv_lim, blk_set) : static_cast<int>(s_kv[j]);
    };
    // A query tile that sees one key tile only (causal: the first query tile;
    // or a single key tile; or a block row with one block): every key its rows
    // see is in that tile, so those rows take D from the tile's own P and dP and
    // their dS goes to the dQ MMA as two 16-bit parts (see the groups below).
    const bool single = n_kv == 1;
    // TMEM columns of key tile j's dP (and, written over it, dS) buffer.
    auto dp_col = [](int j) { return (j & 1) ? Cfg::kColDP1 : Cfg::kColDP; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && (!SPARSE || n_kv > 0)) {
            ptx::prefetch_tmap(&tm_k);
            ptx::prefetch_tmap(&tm_v);
            const uint64_t keep = ptx::policy_evict_last();
            ptx::mbar_arrive_expect_tx(&bar_qdo_full, 2 * TB);
            for (int b = 0; b < G::kNBoxK; ++b) {
                ptx::tma_load_3d(sQ + b * kTileRows * G::kRowBK, &tm_q, &bar_qdo_full, b * G::kBoxK, q_row0, bh);
                ptx::tma_load_3d(sDO + b * kTileRows * G::kRowBK, &tm_do, &bar_qdo_full, b * G::kBoxK, q_row0, bh);
            }
            int k_issued = 0, v_issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int sk = j % RK;
                if (j >= RK && !ptx::mbar_wait(&bar_k_empty[sk], ((j / RK) & 1) ^ 1, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_k_full[sk], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d_hint(sKr + sk * TB + b * kTileRows * G::kRowBK, &tm_k, &bar_k_full[sk], b * G::kBoxK, kv_of(j) * kTileRows, bh_kv, keep);
                k_issued = j + 1;
                const int sv = j % RV;
                if (j >= RV && !ptx::mbar_wait(&bar_v_empty[sv], ((j / RV) & 1) ^ 1, &abort_flag, tmo)) break;
                ptx::mbar_arrive_expect_tx(&bar_v_full[sv], TB);
                for (int b = 0; b < G::kNBoxK; ++b)
                    ptx::tma_load_3d_hint(sVr + sv * TB + b * kTileRows * G::kRowBK, &tm_v, &bar_v_full[sv], b * G::kBoxK, kv_of(j) * kTileRows, bh_kv, keep);
                v_issued = j + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                ptx::mbar_wait_drain(&bar_qdo_full, 0, kDrainNs);
                for (int t = k_issued - 1; t >= 0 && t >= k_issued - RK; --t)
                    ptx::mbar_wait_drain(&bar_k_full[t % RK], (t / RK) & 1, kDrainNs);
                for (int t = v_issued - 1; t >= 0 && t >= v_issued - RV; --t)
                    ptx::mbar_wait_drain(&bar_v_full[t % RV], (t / RV) & 1, kDrainNs);
            }
        }
    } else if (warp == 1 || warp == 10) {
        // ------------------------------------------------ MMA issuers
        // Issuer 0 (warp 1): S(j) for every key tile, each as soon as both
        // groups have read S(j-1).  Issuer 1 (warp 10): dP(0), dP(1); per key
        // tile j dQ += dS(j) K_j, then dP(j+2) (it overwrites dS(j)).  A wait
        // stalls only the thread whose MMAs precede it, so one issuer's MMAs
        // keep the tensor core busy while the other waits.  K_j's slot is
        // released by both S(j) and dQ(j); V_j's by dP(j).
        const int role = warp == 1 ? 0 : 1;
        if (lane == 0 && (!SPARSE || n_kv > 0)) {
            constexpr uint32_t idesc_s = ptx::instr_desc(G::kFmt, 128, 128, false, false);
            constexpr uint32_t idesc_dq = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            const uint32_t q_addr = ptx::smem_addr(sQ);
            const uint32_t do_addr = ptx::smem_addr(sDO);
            auto k_addr = [&](int j) { return ptx::smem_addr(sKr + (j % RK) * TB); };
            auto v_addr = [&](int j) { return ptx::smem_addr(sVr + (j % RV) * TB); };
            auto wait_k = [&](int j) { return ptx::mbar_wait(&bar_k_full[j % RK], (j / RK) & 1, &abort_flag, tmo); };
            bool ok = ptx::mbar_wait(&bar_qdo_full, 0, &abort_flag, tmo);
            if (role == 0) {
                for (int j = 0; ok && j < n_kv; ++j) {
                    // S = Q_i K_j^T   (Eq. 13), into the score columns once S(j-1) is read.
                    if (j > 0 && !ptx::mbar_wait(&bar_s_read, (j - 1) & 1, &abort_flag, tmo)) { ok = false; break; }
                    if (!wait_k(j)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t ka = k_addr(j);
#pragma unroll
                    for (int kk = 0; kk < G::kStepsD; ++kk)
                        ptx::mma_f16_ss(tmem + Cfg::kColS, desc_kmajor<G>(q_addr, kk), desc_kmajor<G>(ka, kk), idesc_s, kk > 0 ? 1u : 0u);
                    ptx::mma_commit(&bar_s_full);
                    ptx::mma_commit(&bar_k_empty[j % RK]);
                }
            } else {
                // dP = dO_i V_j^T   (Eq. 16)
                auto issue_dp = [&](int j) -> bool {
                    if (!ptx::mbar_wait(&bar_v_full[j % RV], (j / RV) & 1, &abort_flag, tmo)) return false;
                    const uint32_t va = v_addr(j);
#pragma unroll
                    for (int kk = 0; kk < G::kStepsD; ++kk)
                        ptx::mma_f16_ss(tmem + dp_col(j), desc_kmajor<G>(do_addr, kk), desc_kmajor<G>(va, kk), idesc_s, kk > 0 ? 1u : 0u);
                    ptx::mma_commit(&bar_dp_full[j & 1]);
                    ptx::mma_commit(&bar_v_empty[j % RV]);
                    return true;
                };
                if (ok) ok = issue_dp(0);
                if (ok && n_kv > 1) ok = issue_dp(1);
                for (int j = 0; ok && j < n_kv; ++j) {
                    // dQ_i += dS K_j   (Eq. 18 without the scale); dS from the dP columns.
                    if (!ptx::mbar_wait(&bar_ds_ready[j & 1], (j >> 1) & 1, &abort_flag, tmo) || !wait_k(j)) { ok = false; break; }
                    ptx::tc_fence_after();
                    const uint32_t ka = k_addr(j);
#pragma unroll
                    for (int kk = 0; kk < G::kStepsRows; ++kk)
                        ptx::mma_f16_ts(tmem + Cfg::kColDQ, tmem + dp_col(j) + a_col(kk), desc_mnmajor<G>(ka, kk), idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
                    if (single) {
                        // dQ += dS_lo K_j: the low parts sit 32 columns after the high parts.
#pragma unroll
                        for (int kk = 0; kk < G::kStepsRows; ++kk)
                            ptx::mma_f16_ts(tmem + Cfg::kColDQ, tmem + Cfg::kColDP + a_col(kk) + 32, desc_mnmajor<G>(ka, kk), idesc_dq, 1u);
                    }
                    ptx::mma_commit(&bar_k_empty[j % RK]);
                    if (j + 2 < n_kv && !issue_dp(j + 2)) { ok = false; break; }
                }
                if (ok) ptx::mma_commit(&bar_dq_done);
            }
            if (!ok) {
                ptx::mma_commit(&bar_drain[role]);
                ptx::mbar_wait_drain(&bar_drain[role], 0, 20000000ull);
            }
        }
    } else {
        // ------------------------------------------------ two P / dS groups
        const int g = (warp - 2) >> 2;                  // key columns [64g, 64g+64)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // query row inside the tile
        const int kc0 = 64 * g;
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        const size_t vrow = static_cast<size_t>(bh) * p.n_pad + q_row0 + r;
        const float l2r = p.l2[vrow];                    // L_i * log2(e) (+inf past N)
        const float dr = p.dvec[vrow];                   // D_i (0 past N)
        bool ok = true;
        if (single) {
            // The rows of this tile see no other key tile (kv_of(0) is the only one), so
            //   D_i = sum_j P_ij dP_ij
            // (the softmax-Jacobian form of rowsum(O o dO), equal to it in exact
            // arithmetic) is formed here from the recomputed P and dP.  Rows that see
            // only a few keys have |dS| of the order of |dP|, and there D taken from
            // the rounded O is not accurate enough; this D keeps sum_j dS_ij = 0.  It
            // is written back for the dK/dV pass.  D uses the fp32 P; dS = P_16 (dP -
            // D), with P_16 the 16-bit P the other passes use, goes to the dQ MMA as
            // two 16-bit parts: hi into the group's first 32 dP columns, lo into the
            // next 32.  With one key tile there is nothing to overlap, so both S and dP
            // are awaited first.  Every elementwise thread reaches the named barrier
            // below exactly once, also when a wait gave up.
            const int kv = kv_of(0);
            const bool diag = p.causal && (kv == q_tile);
            const int kv_valid = p.Nk - kv * kTileRows - kc0;
            uint32_t pk[32];
            bool got = __all_sync(0xffffffffu, ptx::mbar_wait(&bar_s_full, 0, &abort_flag, tmo) &&
                                                   ptx::mbar_wait(&bar_dp_full[0], 0, &abort_flag, tmo));
            float part = 0.f;
            if (got) {
                ptx::tc_fence_after();
                const float2 sl2v = make_float2(sl2, sl2), nl2v = make_float2(-l2r, -l2r);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t us[32], ud[32];
                    ptx::tmem_ld32(lane_base + Cfg::kColS + kc0 + 32 * h, us);
                    ptx::tmem_ld32(lane_base + Cfg::kColDP + kc0 + 32 * h, ud);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        const int cc = 32 * h + c;
                        const float2 a = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, nl2v);
                        const float p0 = ((diag && kc0 + cc > r) || cc >= kv_valid) ? 0.f : ptx::ex2_approx(a.x);
                        const float p1 = ((diag && kc0 + cc + 1 > r) || cc + 1 >= kv_valid) ? 0.f : ptx::ex2_approx(a.y);
                        pk[cc >> 1] = G::pack2(p0, p1);
                        part = fmaf(p0, __uint_as_float(ud[c]), part);
                        part = fmaf(p1, __uint_as_float(ud[c + 1]), part);
                    }
                }
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_s_read);
            }
            // Both groups' partial sums meet in the V ring's second slot (unused: this
            // CTA loads one key tile).
            float* s_dpart = reinterpret_cast<float*>(sVr + TB);
            s_dpart[g * kTileRows + r] = part;
            asm volatile("bar.sync 3, 256;" ::: "memory");
            if (!got) {
                ok = false;
            } else {
                const float dfull = s_dpart[r] + s_dpart[kTileRows + r];
                if (g == 0 && q_row0 + r < p.N) p.dvec[vrow] = dfull;
                const float2 ndv = make_float2(-dfull, -dfull);
                uint32_t lo_a[16];
                {
                    uint32_t ud[32], hi[16];
                    ptx::tmem_ld32(lane_base + Cfg::kColDP + kc0, ud);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        float2 pp, hv;
                        G::unpack2(pk[c >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c]), __uint_as_float(ud[c + 1])), ndv));
                        hi[c >> 1] = G::pack2(ds.x, ds.y);
                        G::unpack2(hi[c >> 1], hv.x, hv.y);
                        lo_a[c >> 1] = G::pack2(ds.x - hv.x, ds.y - hv.y);
                    }
                    ptx::tmem_st16(lane_base + Cfg::kColDP + kc0, hi);          // dS_hi, values 0..31
                }
                {
                    uint32_t ud[32], hi[16], lo[16];
                    ptx::tmem_ld32(lane_base + Cfg::kColDP + kc0 + 32, ud);
                    ptx::tmem_wait_ld();
                    ptx::tmem_st16(lane_base + Cfg::kColDP + kc0 + 32, lo_a);     // dS_lo, values 0..31
#pragma unroll
                    for (int c = 0; c < 32; c += 2) {
                        float2 pp, hv;
                        G::unpack2(pk[(32 + c) >> 1], pp.x, pp.y);
                        const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c]), __uint_as_float(ud[c + 1])), ndv));
                        hi[c >> 1] = G::pack2(ds.x, ds.y);
                        G::unpack2(hi[c >> 1], hv.x, hv.y);
                        lo[c >> 1] = G::pack2(ds.x - hv.x, ds.y - hv.y);
                    }
                    ptx::tmem_st16(lane_base + Cfg::kColDP + kc0 + 16, hi);     // dS_hi, values 32..63
                    ptx::tmem_st16(lane_base + Cfg::kColDP + kc0 + 48, lo);     // dS_lo, values 32..63
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_ds_ready[0]);
            }
        }
        for (int j = 0; !single && j < n_kv; ++j) {
            const int kv = kv_of(j);
            const bool diag = p.causal && (kv == q_tile);
            const int kv_valid = p.Nk - kv * kTileRows - kc0;  // this group's key columns < Nk
            // ---- P = exp2(S * scale*log2(e) - L*log2(e))   (Eq. 14)
            if (!ptx::mbar_wait(&bar_s_full, j & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pk[32];
            {
                uint32_t us[64];
                ptx::tmem_ld32(lane_base + Cfg::kColS + kc0, *reinterpret_cast<uint32_t(*)[32]>(us));
                ptx::tmem_ld32(lane_base + Cfg::kColS + kc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(us + 32));
                ptx::tmem_wait_ld();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_s_read);
                const float2 sl2v = make_float2(sl2, sl2), nl2v = make_float2(-l2r, -l2r);
                if (diag || kv_valid < 64) {
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float2 a = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, nl2v);
                        float p0 = ptx::ex2_approx(a.x), p1 = ptx::ex2_approx(a.y);
                        if ((diag && kc0 + c > r) || c >= kv_valid) p0 = 0.f;
                        if ((diag && kc0 + c + 1 > r) || c + 1 >= kv_valid) p1 = 0.f;
                        pk[c >> 1] = G::pack2(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 64; c += 2) {
                        const float2 a = ptx::fma2(make_float2(__uint_as_float(us[c]), __uint_as_float(us[c + 1])), sl2v, nl2v);
                        pk[c >> 1] = G::pack2(ptx::ex2_approx(a.x), ptx::ex2_approx(a.y));
                    }
                }
            }
            // ---- dS = P o (dP - D)   (Eq. 17) -> TMEM over dP
            if (!ptx::mbar_wait(&bar_dp_full[j & 1], (j >> 1) & 1, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            const uint32_t dpc = dp_col(j);
            uint32_t dk[32];
            {
                uint32_t ud[64];
                ptx::tmem_ld32(lane_base + dpc + kc0, *reinterpret_cast<uint32_t(*)[32]>(ud));
                ptx::tmem_ld32(lane_base + dpc + kc0 + 32, *reinterpret_cast<uint32_t(*)[32]>(ud + 32));
                ptx::tmem_wait_ld();
                const float2 ndv = make_float2(-dr, -dr);
#pragma unroll
                for (int c = 0; c < 64; c += 2) {
                    float2 pp;
                    G::unpack2(pk[c >> 1], pp.x, pp.y);
                    const float2 ds = ptx::mul2(pp, ptx::add2(make_float2(__uint_as_float(ud[c]), __uint_as_float(ud[c + 1])), ndv));
                    dk[c >> 1] = G::pack2(ds.x, ds.y);
                }
            }
            // dS -> this group's own columns of the dP buffer [64g, 64g + 32), already read.
            ptx::tmem_st32(lane_base + dpc + kc0, dk);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_ds_ready[j & 1]);
        }
        // ---------------- epilogue (group 0): dQ * scale -> shared memory -> TMA store.
        if (g == 0) {
            if (ok && (!SPARSE || n_kv > 0)) ok = ptx::mbar_wait(&bar_dq_done, 0, &abort_flag, tmo);
            if (ok) {
                ptx::tc_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
                    uint32_t u[16];
                    if (SPARSE && n_kv == 0) {
#pragma unroll
                        for (int c = 0; c < 16; ++c) u[c] = 0u;
                    } else {
                        ptx::tmem_ld16(lane_base + Cfg::kColDQ + c0, u);
                        ptx::tmem_wait_ld();
                    }
#pragma unroll
                    for (int h8 = 0; h8 < 2; ++h8) {
                        const int cc = c0 + 8 * h8;
                        if (cc < D) {
                            const float* f = reinterpret_cast<const float*>(u) + 8 * h8;
                            const float s = p.scale;
                            uint4 w;
                            w.x = G::pack2(f[0] * s, f[1] * s);
                            w.y = G::pack2(f[2] * s, f[3] * s);
                            w.z = G::pack2(f[4] * s, f[5] * s);
                            w.w = G::pack2(f[6] * s, f[7] * s);
                            *reinterpret_cast<uint4*>(sQ + kmajor_chunk_offset<G>(r, cc)) = w;
                        }
                    }
                }
                ptx::fence_async_smem();
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (ok && (threadIdx.x & 127) == 64) {
                for (int bx = 0; bx < G::kNBoxK; ++bx)
                    ptx::tma_store_3d(&tm_dq, sQ + bx * kTileRows * G::kRowBK, bx * G::kBoxK, q_row0, bh);
                ptx::tma_store_commit();
                ptx::tma_store_wait_all();
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
