// fa2_bwd32.cuh -- the FlashAttention-2 backward pass for fp32 inputs, on
// TF32 tensor cores (tcgen05.mma kind::tf32), for sm_100a.
//
// Same equations (CS336 A2 Systems handout section 4.2.2, Eqs. 13-19) and the
// same two-pass organisation as the 16-bit kernels in fa2_bwd.cuh: a pass that
// owns a key/value tile and accumulates its dK and dV, then a pass that owns a
// query tile and accumulates its dQ (the handout's Algorithm 2, section
// 4.2.3), after a pre-processing kernel of its own.  Three things differ with
// 4-byte elements:
//
//  * A TF32 operand contracted over tile rows (dO and Q in the dK/dV pass, K
//    in the dQ pass) must sit in shared memory with the 128-byte swizzle of
//    32-byte atoms, which the contraction over d cannot read.  Those operands
//    are staged twice, once per layout (two TMA copies of the same rows).
//  * A 128-row tile is up to 64 KB, so the streamed operand arrives in
//    sub-tiles of W rows: the largest W in {128, 64, 32, 16} that leaves room
//    for two pipeline stages beside the two resident 128-row tiles.
//  * P and dS stay fp32 in tensor memory, one column per element, written over
//    the scores they came from; the next MMA reads them there as TF32.
//
// Every TF32 operand is rounded to nearest before the tensor core sees it: the
// pre-processing kernel writes rounded copies of q, k, v and dout into the
// workspace (the kernels' TMA loads read those), and P and dS are rounded as
// they are written to tensor memory.  The tensor core itself would drop the 13
// low bits of an fp32 operand, a biased error that puts a few gradient
// elements past the 2e-3 tolerance.  D = rowsum(O o dO) is formed from the
// rounded dO, the dO every dP entry is computed from, so that D_i stays equal
// to sum_j P_ij dP_ij as the kernels compute them.
//
// Both kernels use 6 warps: 0 TMA producer, 1 MMA issuer (one thread), 2-5
// one elementwise warpgroup.  The thread holding TMEM lane t owns row t of the
// CTA's 128-row tile and all W columns of the current sub-tile.
#pragma once

#include <cstdint>

#include "fa2_bwd.cuh"

namespace fa2 {

template <int D>
struct Bwd32Cfg {
    using G = TileGeom<4, D>;
    static constexpr int kThreads = 192;
    // dK/dV pass at d <= 64, where its elementwise work outweighs the MMAs: two
    // P / dS warpgroups take alternate query sub-tiles (S^T and dP^T double
    // buffered in TMEM), so one group's exponentials overlap the other's MMAs.
    static constexpr int kGroupsKV = D <= 64 ? 2 : 1;
    static constexpr int kThreadsKV = 64 + 128 * kGroupsKV;
    // dQ pass likewise at d <= 32: two warpgroups on alternate key sub-tiles of
    // 64 rows (one group took 128-row sub-tiles; at d = 64, with Q and dO in
    // TMEM, two groups measured 1-3 % slower).
    static constexpr int kGroupsQ = D <= 32 ? 2 : 1;
    static constexpr int kThreadsQ = 64 + 128 * kGroupsQ;
    // 227 KB minus the 1024-byte alignment pad and the static shared memory.
    static constexpr int kBudget = 227 * 1024 - 1024 - 1024;
    __host__ __device__ static constexpr int tile_k(int rows) { return G::kNBoxK * rows * G::kRowBK; }
    __host__ __device__ static constexpr int tile_mn(int rows) { return G::kNBoxMN * rows * G::kRowBMN; }
    static constexpr int kResident = 2 * tile_k(kTileRows);
    // dK/dV pass at d = 64 and 128: K sits in tensor memory (the S^T = K Q^T MMA
    // reads its A operand there), so only V is resident in shared memory.  At
    // d = 128 that leaves room for 64-row query sub-tiles (part-staged, below)
    // instead of 16: the pass was bound by the tcgen05 instruction pipe, the
    // narrow S^T / dP^T MMAs (N = W) being most of its instructions.  At d = 64
    // it leaves room for a third stage, which the two groups need (sub-tile
    // i + 2 loads while i and i + 1 are being worked on).
    static constexpr bool kKInTmem = (D == 64 || D == 128);
    static constexpr int kResidentKV = (kKInTmem ? 1 : 2) * tile_k(kTileRows);
    // dQ pass at d = 64 and 128, likewise: Q and dO in tensor memory (the A
    // operands of S = Q K^T and dP = dO V^T), nothing resident in shared memory,
    // and key sub-tiles of 128 rows instead of 64 (d = 64), 64 instead of 32
    // (d = 128).
    static constexpr bool kQInTmem = (D == 64 || D == 128);
    static constexpr int kResidentQ = kQInTmem ? 0 : 2 * tile_k(kTileRows);
    __host__ __device__ static constexpr int stages_for(int stage_bytes, int resident = kResident) {
        const int s = (kBudget - resident) / stage_bytes;
        return s > 4 ? 4 : s;
    }
    // dK/dV pass, per stage: W query rows of Q and of dO, each K-major and MN-major.
    __host__ __device__ static constexpr int kv_stage(int w) { return 2 * tile_k(w) + 2 * tile_mn(w); }
    // dQ pass, per stage: W key rows of K (K-major and MN-major) and of V (K-major).
    __host__ __device__ static constexpr int q_stage(int w) { return 2 * tile_k(w) + tile_mn(w); }
    __host__ __device__ static constexpr int pick_kv() {
        for (int w = kTileRows; w > 16; w /= 2)
            if (stages_for(kv_stage(w), kResidentKV) >= 2) return w;
        return 16;
    }
    __host__ __device__ static constexpr int pick_q() {
        for (int w = kTileRows; w > 16; w /= 2)
            if (stages_for(q_stage(w), kResidentQ) >= 2) return w;
        return 16;
    }
    // At most 64 query rows per dK/dV sub-tile: with 128 (d = 16, 32) a thread's
    // P^T row of W fp32 values spilled, and the pass ran 10 % slower, same bits.
    // dK/dV pass at d = 128 (K in TMEM): sub-tiles of 64 query rows in a single
    // stage whose four parts (Q and dO, each K-major and MN-major) are refilled
    // one by one as soon as the one MMA group that reads each has finished, plus a
    // second slot for Q K-major, the part each sub-tile needs first.  Two whole
    // stages of 64 rows do not fit beside V; 32-row sub-tiles left the tcgen05
    // instruction pipe the busiest unit of the pass.
    static constexpr bool kPartStaged = D == 128;
    static constexpr int kWkv = kPartStaged ? 64 : (pick_kv() > 64 ? 64 : pick_kv());
    static constexpr int kStKV = kPartStaged ? 1 : stages_for(kv_stage(kWkv), kResidentKV);
    static constexpr int kWq = kGroupsQ == 2 ? 64 : pick_q();
    static constexpr int kStQ = stages_for(q_stage(kWq), kResidentQ);
    static_assert((kPartStaged || kStKV >= 2) && kStQ >= 2, "shared memory too small for two pipeline stages");
    static constexpr int kSmemKV = 1024 + kResidentKV +
        (kPartStaged ? 3 * tile_k(kWkv) + 2 * tile_mn(kWkv) : kStKV * kv_stage(kWkv));
    static_assert(kSmemKV <= 227 * 1024 - 1024, "dK/dV pass shared memory over the limit");
    static constexpr int kSmemQ = 1024 + kResidentQ + kStQ * q_stage(kWq);
    static constexpr uint32_t kTmemCols = 512;
    // dK/dV pass: S^T | dP^T | dV | dK.   dQ pass: S | dP | dQ.
    static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 384, kColDQ = 256;
    // dK/dV pass, general: S^T (per group) | dP^T (per group) | [K] | dV | dK.
    static constexpr uint32_t kColDPkv = (kKInTmem || kGroupsKV == 2) ? kGroupsKV * kWkv : kColDP;
    static constexpr uint32_t kColKT = 2 * kGroupsKV * kWkv;
    static constexpr uint32_t kColDVkv = kKInTmem ? kColKT + G::kStepsD * G::kKStep : kColDV;
    static constexpr uint32_t kColDKkv = kKInTmem ? kColDVkv + G::kNOut : kColDK;
    static_assert(kColDPkv + kGroupsKV * kWkv <= (kKInTmem ? kColKT : kColDV) && kColDKkv + G::kNOut <= kTmemCols,
                  "dK/dV pass columns overlap or exceed TMEM");
    // dQ pass, general: S (per group) | dP (per group) | dQ | [Q | dO].
    static constexpr uint32_t kColDPq = kQInTmem ? kGroupsQ * kWq : kColDP;
    static constexpr uint32_t kColDQq = kQInTmem ? 2 * kGroupsQ * kWq : kColDQ;
    static constexpr uint32_t kColQT = kColDQq + G::kNOut, kColDOT = kColQT + G::kStepsD * G::kKStep;
    static_assert(kGroupsQ * kWq <= kColDPq && kColDPq + kGroupsQ * kWq <= kColDQq, "dQ pass S / dP columns overlap");
    static_assert(!kQInTmem || kColDOT + G::kStepsD * G::kKStep <= kTmemCols, "dQ pass columns exceed TMEM");
};

// ------------------------------------------------------------------ pre-processing

// One warp per query row (8 rows per block): TF32-rounded copies of the q and
// dout rows, D_i = sum_t round(dO_it) O_it, and L_i * log2(e); rows past N (up
// to the padded length) get D = 0 and L = +inf.
template <int D>
__global__ void __launch_bounds__(256)
fa2_bwd32_pre_kernel(const float* __restrict__ q, const float* __restrict__ o,
                     const float* __restrict__ dout, const float* __restrict__ lse,
                     float* __restrict__ qr, float* __restrict__ dor, float* __restrict__ l2,
                     float* __restrict__ dvec, int N, int n_pad, long long rows_total) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
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
    // 16-byte accesses (D is a multiple of 4): a lane takes columns 4e .. 4e + 3.
    const float4* q4 = reinterpret_cast<const float4*>(q + base);
    const float4* o4 = reinterpret_cast<const float4*>(o + base);
    const float4* g4 = reinterpret_cast<const float4*>(dout + base);
    float4* qr4 = reinterpret_cast<float4*>(qr + base);
    float4* dor4 = reinterpret_cast<float4*>(dor + base);
    auto rna = [](float x) { return __uint_as_float(ptx::to_tf32_rna(x)); };
    for (int e = lane; e < D / 4; e += 32) {
        const float4 gv = __ldg(g4 + e), qv = __ldg(q4 + e), ov = __ldg(o4 + e);
        const float4 g = make_float4(rna(gv.x), rna(gv.y), rna(gv.z), rna(gv.w));
        dor4[e] = g;
        qr4[e] = make_float4(rna(qv.x), rna(qv.y), rna(qv.z), rna(qv.w));
        acc += ov.x * g.x + ov.y * g.y + ov.z * g.z + ov.w * g.w;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
        dvec[row] = acc;
        l2[row] = lse[static_cast<size_t>(bh) * N + n] * 1.4426950408889634f;
    }
}

// TF32-rounded copy of an fp32 tensor (k or v: [B * H_kv][N][d]), n4 float4s.
__global__ void __launch_bounds__(256)
fa2_round_tf32_kernel(const float4* __restrict__ in, float4* __restrict__ out, size_t n4) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n4;
         i += static_cast<size_t>(gridDim.x) * blockDim.x) {
        float4 x = in[i];
        x.x = __uint_as_float(ptx::to_tf32_rna(x.x));
        x.y = __uint_as_float(ptx::to_tf32_rna(x.y));
        x.z = __uint_as_float(ptx::to_tf32_rna(x.z));
        x.w = __uint_as_float(ptx::to_tf32_rna(x.w));
        out[i] = x;
    }
}

// W consecutive TMEM columns of this warp's 32 lanes, one 32-bit word each.
template <int W>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&u)[W]) {
    if constexpr (W == 16) {
        ptx::tmem_ld16(taddr, u);
    } else {
#pragma unroll
        for (int c = 0; c < W; c += 32)
            ptx::tmem_ld32(taddr + c, *reinterpret_cast<uint32_t(*)[32]>(u + c));
    }
}

template <int W>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&u)[W]) {
    if constexpr (W == 16) {
        ptx::tmem_st16(taddr, u);
    } else {
#pragma unroll
        for (int c = 0; c < W; c += 32)
            ptx::tmem_st32(taddr + c, *reinterpret_cast<const uint32_t(*)[32]>(u + c));
    }
}

// P (fp32 bit patterns in `pu`) rounded to TF32 -> W TMEM columns at `col`;
// `pu` keeps the unrounded values for dS.
template <int W>
__device__ __forceinline__ void bwd32_store_p(uint32_t col, const uint32_t (&pu)[W]) {
    constexpr int C = W < 32 ? W : 32;
#pragma unroll
    for (int c0 = 0; c0 < W; c0 += C) {
        uint32_t u[C];
#pragma unroll
        for (int c = 0; c < C; ++c) u[c] = ptx::to_tf32_rna(__uint_as_float(pu[c0 + c]));
        tmem_st_cols<C>(col + c0, u);
    }
}

// dS = P o (dP - D) over W columns held in TMEM at `dp_col`, rounded to TF32
// and written back in place; P (fp32 bit patterns) is in `pu`, D per column or
// per row from `dval`.
template <int W, class DOf>
__device__ __forceinline__ void bwd32_ds_inplace(uint32_t dp_col, const uint32_t (&pu)[W], DOf dval) {
    constexpr int C = W < 32 ? W : 32;
#pragma unroll
    for (int c0 = 0; c0 < W; c0 += C) {
        uint32_t u[C];
        tmem_ld_cols<C>(dp_col + c0, u);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < C; ++c)
            u[c] = ptx::to_tf32_rna(__uint_as_float(pu[c0 + c]) * (__uint_as_float(u[c]) - dval(c0 + c)));
        tmem_st_cols<C>(dp_col + c0, u);
    }
    ptx::tmem_wait_st();
}

// 128 x D fp32 accumulator in TMEM (this thread's row r) times `mul` -> the
// K-major staging layout of an fp32 tile in shared memory; zeros instead when
// `zero` (nothing was accumulated).
template <class G>
__device__ __forceinline__ void bwd32_stage_rows(uint32_t acc_col, int r, float mul, uint8_t* stage,
                                                 bool zero = false) {
#pragma unroll
    for (int c0 = 0; c0 < G::kNOut; c0 += 16) {
        uint32_t u[16] = {};
        if (!zero) {
            ptx::tmem_ld16(acc_col + c0, u);
            ptx::tmem_wait_ld();
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
            const int col = c0 + 4 * q4;
            if (col < G::kD) {
                uint4 w;
                w.x = __float_as_uint(__uint_as_float(u[4 * q4 + 0]) * mul);
                w.y = __float_as_uint(__uint_as_float(u[4 * q4 + 1]) * mul);
                w.z = __float_as_uint(__uint_as_float(u[4 * q4 + 2]) * mul);
                w.w = __float_as_uint(__uint_as_float(u[4 * q4 + 3]) * mul);
                *reinterpret_cast<uint4*>(stage + kmajor_chunk_offset<G>(r, col)) = w;
            }
        }
    }
}

// ------------------------------------------------------------------ dK / dV pass

// One CTA per (key tile j, head); K_j and V_j stay resident, the query rows
// that see key tile j stream through in sub-tiles of W rows.  Per sub-tile
// the MMA issuer runs S^T = K Q^T, dP^T = V dO^T, dV += P^T dO, dK += dS^T Q,
// issuing the next sub-tile's S^T right after dV and its dP^T right after dK.
// With a block mask (SPARSE) only the sub-tiles of query tiles whose block with
// key tile j is set are visited, found by each thread walking the mask column.
template <int D, bool SPARSE = false>
__global__ void __launch_bounds__(Bwd32Cfg<D>::kThreadsKV, 1)
fa2_bwd32_dkdv_kernel(const __grid_constant__ CUtensorMap tm_qk, const __grid_constant__ CUtensorMap tm_qmn,
                      const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_dok, const __grid_constant__ CUtensorMap tm_domn,
                      const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv,
                      const BwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = Bwd32Cfg<D>;
    using G = typename Cfg::G;
    constexpr int W = Cfg::kWkv;
    constexpr int ST = Cfg::kStKV;
    constexpr int TK = Cfg::tile_k(kTileRows);
    constexpr int SK = Cfg::tile_k(W);
    constexpr int SM = Cfg::tile_mn(W);
    constexpr int SB = Cfg::kv_stage(W);

    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar_kv_full, bar_full[ST], bar_empty[ST];
    constexpr int NG = Cfg::kGroupsKV;                  // P / dS warpgroups (buffers)
    static_assert(NG == 1 || (!Cfg::kPartStaged && NG * W <= 128), "S^T / dP^T buffers exceed their TMEM columns");
    __shared__ uint64_t bar_s_full[NG], bar_dp_full[NG], bar_p_ready[NG], bar_ds_ready[NG], bar_dkv_full, bar_drain;
    __shared__ uint64_t bar_kt_ready;                   // K written to tensor memory (KT)
    // Part-staged (PP): full / empty barrier per part slot: Q K-major slots 0 and
    // 1, then dO K-major, Q MN-major, dO MN-major.
    __shared__ uint64_t bar_pf[5], bar_pe[5];
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    __shared__ int s_cnt;                               // block-sparse: query sub-tiles per head

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    constexpr bool KT = Cfg::kKInTmem;
    uint8_t* sK = smem;                                 // unused when K is in tensor memory
    uint8_t* sV = KT ? smem : sK + TK;
    uint8_t* sStage = sV + TK;
    // dK is staged for its store where K was, or in the (then idle) first stage.
    uint8_t* sDK = KT ? sStage : sK;
    // Stage s: Q (K-major) | dO (K-major) | Q (MN-major) | dO (MN-major).
    // Part-staged: Q (K-major) slot 0 | slot 1 | dO (K-major) | Q (MN-major) | dO (MN-major).
    constexpr bool PP = Cfg::kPartStaged;
    constexpr int kPartQk = 0, kPartDok = 1, kPartQmn = 2, kPartDomn = 3;
    auto pp_slot = [](int part, int it) { return part == kPartQk ? (it & 1) : part + 1; };
    auto pp_phase = [](int part, int it) -> uint32_t { return static_cast<uint32_t>(part == kPartQk ? it >> 1 : it) & 1u; };
    auto pp_addr = [&](int part, int it) -> uint8_t* {
        return part == kPartQk ? sStage + (it & 1) * SK
             : part == kPartDok ? sStage + 2 * SK
             : part == kPartQmn ? sStage + 3 * SK : sStage + 3 * SK + SM;
    };
    auto st_qk = [&](int s) { return sStage + s * SB; };
    auto st_dok = [&](int s) { return sStage + s * SB + SK; };
    auto st_qmn = [&](int s) { return sStage + s * SB + 2 * SK; };
    auto st_domn = [&](int s) { return sStage + s * SB + 2 * SK + SM; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: (key tile j, key/value head).  Key tile j is seen by query
    // rows >= 128 j (causal) of each of the `group` query heads sharing this
    // key/value head, whose dK and dV sum over all of them; small j carries
    // the most work and is issued first.
    const int item = blockIdx.x;
    const int kv_tile = item / p.BH_kv;
    const int bh = item - kv_tile * p.BH_kv;            // key/value head
    const int kv_row0 = kv_tile * kTileRows;
    const int n_sub = (p.N + W - 1) / W;                // query sub-tiles
    const int sub_begin = p.causal ? kv_row0 / W : 0;
    constexpr int R = kTileRows / W;                    // sub-tiles per 128-row tile
    // Block-sparse: query tiles i_begin + t (t < n_col) whose block is set.
    const int i_begin = p.causal ? kv_tile : 0;
    const int n_col = p.n_tiles > i_begin ? p.n_tiles - i_begin : 0;
    auto blk_set = [&](int t) {
        return __ldg(p.block_mask + static_cast<size_t>(i_begin + t) * p.n_tiles_k + kv_tile) != 0;
    };
    if (SPARSE && warp == 0) {
        int c = 0;
        for (int base = 0; base < n_col; base += 32)
            c += __popc(__ballot_sync(0xffffffffu, base + lane < n_col && blk_set(base + lane)));
        // R sub-tiles per set query tile; the last query tile's end at n_sub.
        const bool last = n_col > 0 && blk_set(n_col - 1);
        if (lane == 0) s_cnt = c * R - (last ? p.n_tiles * R - n_sub : 0);
    }
    MaskWalk walker;

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_kv_full, 1);
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&bar_full[s], 1);
            ptx::mbar_init(&bar_empty[s], 1);
        }
        for (int b = 0; b < NG; ++b) {
            ptx::mbar_init(&bar_s_full[b], 1);
            ptx::mbar_init(&bar_dp_full[b], 1);
            ptx::mbar_init(&bar_p_ready[b], 4);
            ptx::mbar_init(&bar_ds_ready[b], 4);
        }
        ptx::mbar_init(&bar_dkv_full, 1);
        ptx::mbar_init(&bar_drain, 1);
        ptx::mbar_init(&bar_kt_ready, 4);
        for (int b = 0; b < 5; ++b) {
            ptx::mbar_init(&bar_pf[b], 1);
            ptx::mbar_init(&bar_pe[b], 1);
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
    // Sub-tiles per query head; none when no query reaches this key tile
    // (causal, keys longer than queries; or an empty block column): then
    // dK = dV = 0 is written.
    const int n_q = SPARSE ? s_cnt : (n_sub > sub_begin ? n_sub - sub_begin : 0);
    const int n_it = n_q * p.group;                     // (query head, sub-tile) steps
    auto q_row_walk = [&](MaskWalk& w, int it) {
        const int g = it % n_q;
        if (!SPARSE) return (sub_begin + g) * W;
        return ((i_begin + w.at(g / R, n_col, blk_set)) * R + g % R) * W;
    };
    auto q_row_of = [&](int it) { return q_row_walk(walker, it); };
    auto q_head_of = [&](int it) { return (bh / p.H_kv) * p.H + (bh % p.H_kv) * p.group + it / n_q; };

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_it > 0) {
            ptx::prefetch_tmap(&tm_qk);
            ptx::prefetch_tmap(&tm_qmn);
            ptx::prefetch_tmap(&tm_dok);
            ptx::prefetch_tmap(&tm_domn);
            ptx::mbar_arrive_expect_tx(&bar_kv_full, (KT ? 1 : 2) * TK);
            for (int b = 0; b < G::kNBoxK; ++b) {
                if (!KT) ptx::tma_load_3d(sK + b * kTileRows * G::kRowBK, &tm_k, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
                ptx::tma_load_3d(sV + b * kTileRows * G::kRowBK, &tm_v, &bar_kv_full, b * G::kBoxK, kv_row0, bh);
            }
            if constexpr (PP) {
                // The four parts stream independently, each into its slot(s) as
                // soon as the MMA group that last read the slot has finished.
                MaskWalk walk[4];
                int nxt[4] = {0, 0, 0, 0};              // sub-tiles issued, per part
                uint32_t spins = 0;
                uint64_t t_idle = 0;
                while (nxt[0] < n_it || nxt[1] < n_it || nxt[2] < n_it || nxt[3] < n_it) {
                    bool moved = false;
#pragma unroll
                    for (int part = 0; part < 4; ++part) {
                        const int it = nxt[part];
                        if (it >= n_it) continue;
                        const int depth = part == kPartQk ? 2 : 1;
                        const int b = pp_slot(part, it);
                        if (it >= depth && !ptx::mbar_test_wait(&bar_pe[b], pp_phase(part, it) ^ 1u)) continue;
                        const int row0 = q_row_walk(walk[part], it);
                        const int qh = q_head_of(it);
                        uint8_t* dst = pp_addr(part, it);
                        if (part == kPartQk || part == kPartDok) {
                            ptx::mbar_arrive_expect_tx(&bar_pf[b], SK);
                            for (int bx = 0; bx < G::kNBoxK; ++bx)
                                ptx::tma_load_3d(dst + bx * W * G::kRowBK, part == kPartQk ? &tm_qk : &tm_dok, &bar_pf[b],
                                                 bx * G::kBoxK, row0, qh);
                        } else {
                            ptx::mbar_arrive_expect_tx(&bar_pf[b], SM);
                            for (int bx = 0; bx < G::kNBoxMN; ++bx)
                                ptx::tma_load_3d(dst + bx * W * G::kRowBMN, part == kPartQmn ? &tm_qmn : &tm_domn, &bar_pf[b],
                                                 bx * G::kBoxMN, row0, qh);
                        }
                        nxt[part] = it + 1;
                        moved = true;
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
                    constexpr uint64_t kDrainNs = 20000000ull;
                    ptx::mbar_wait_drain(&bar_kv_full, 0, kDrainNs);
                    for (int part = 0; part < 4; ++part) {
                        const int depth = part == kPartQk ? 2 : 1;
                        for (int t = nxt[part] - 1; t >= 0 && t >= nxt[part] - depth; --t)
                            ptx::mbar_wait_drain(&bar_pf[pp_slot(part, t)], pp_phase(part, t), kDrainNs);
                    }
                }
            } else {
            int issued = 0;
            for (int it = 0; it < n_it; ++it) {
                const int s = it % ST;
                if (it >= ST && !ptx::mbar_wait(&bar_empty[s], ((it / ST) & 1) ^ 1, &abort_flag, tmo)) break;
                const int row0 = q_row_of(it);
                const int qh = q_head_of(it);
                ptx::mbar_arrive_expect_tx(&bar_full[s], SB);
                for (int b = 0; b < G::kNBoxK; ++b) {
                    ptx::tma_load_3d(st_qk(s) + b * W * G::kRowBK, &tm_qk, &bar_full[s], b * G::kBoxK, row0, qh);
                    ptx::tma_load_3d(st_dok(s) + b * W * G::kRowBK, &tm_dok, &bar_full[s], b * G::kBoxK, row0, qh);
                }
                for (int b = 0; b < G::kNBoxMN; ++b) {
                    ptx::tma_load_3d(st_qmn(s) + b * W * G::kRowBMN, &tm_qmn, &bar_full[s], b * G::kBoxMN, row0, qh);
                    ptx::tma_load_3d(st_domn(s) + b * W * G::kRowBMN, &tm_domn, &bar_full[s], b * G::kBoxMN, row0, qh);
                }
                issued = it + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                ptx::mbar_wait_drain(&bar_kv_full, 0, kDrainNs);
                for (int t = issued - 1; t >= 0 && t >= issued - ST; --t)
                    ptx::mbar_wait_drain(&bar_full[t % ST], (t / ST) & 1, kDrainNs);
            }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n_it > 0) {
            constexpr uint32_t idesc_s = ptx::instr_desc(G::kFmt, 128, W, false, false);
            constexpr uint32_t idesc_kv = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            const uint32_t k_addr = ptx::smem_addr(sK);
            const uint32_t v_addr = ptx::smem_addr(sV);
            // S^T = K_j Q_i^T   (Eq. 13, transposed: rows are keys)
            // Part-staged: wait for one part, and release it after its MMAs.
            auto wait_part = [&](int part, int it) -> bool {
                if constexpr (PP) {
                    if (!ptx::mbar_wait(&bar_pf[pp_slot(part, it)], pp_phase(part, it), &abort_flag, tmo)) return false;
                    ptx::tc_fence_after();
                }
                return true;
            };
            auto release_part = [&](int part, int it) {
                if constexpr (PP) ptx::mma_commit(&bar_pe[pp_slot(part, it)]);
            };
            auto issue_s = [&](int it) -> bool {
                const int s = it % ST;
                if constexpr (PP) {
                    if (!wait_part(kPartQk, it)) return false;
                } else {
                    if (!ptx::mbar_wait(&bar_full[s], (it / ST) & 1, &abort_flag, tmo)) return false;
                    ptx::tc_fence_after();
                }
                const uint32_t qa = ptx::smem_addr(PP ? pp_addr(kPartQk, it) : st_qk(s));
                const int b = it % NG;
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk) {
                    if constexpr (KT)
                        ptx::mma_tf32_ts(tmem + Cfg::kColS + b * W, tmem + Cfg::kColKT + kk * G::kKStep, desc_kmajor<G>(qa, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_tf32_ss(tmem + Cfg::kColS + b * W, desc_kmajor<G>(k_addr, kk), desc_kmajor<G>(qa, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bar_s_full[b]);
                release_part(kPartQk, it);
                return true;
            };
            // dP^T = V_j dO_i^T   (Eq. 16, transposed); the stage is already full
            // (part-staged: its dO K-major part is waited for here).
            auto issue_dp = [&](int it) -> bool {
                if (!wait_part(kPartDok, it)) return false;
                const uint32_t da = ptx::smem_addr(PP ? pp_addr(kPartDok, it) : st_dok(it % ST));
                const int b = it % NG;
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk)
                    ptx::mma_tf32_ss(tmem + Cfg::kColDPkv + b * W, desc_kmajor<G>(v_addr, kk), desc_kmajor<G>(da, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                ptx::mma_commit(&bar_dp_full[b]);
                release_part(kPartDok, it);
                return true;
            };
            bool ok = ptx::mbar_wait(&bar_kv_full, 0, &abort_flag, tmo);
            if (KT && ok) ok = ptx::mbar_wait(&bar_kt_ready, 0, &abort_flag, tmo);
            for (int i = 0; ok && i < NG && i < n_it; ++i) {
                ok = issue_s(i);
                if (ok) ok = issue_dp(i);
            }
            // Sub-tile it + NG reuses the buffers of sub-tile it: its S^T follows
            // dV(it), its dP^T follows dK(it) (the MMAs that read them).
            for (int it = 0; ok && it < n_it; ++it) {
                const int s = it % ST;
                const int b = it % NG;
                const uint32_t ph = static_cast<uint32_t>(it / NG) & 1u;
                // dV_j += P^T dO_i   (Eq. 15); P^T read from the score columns.
                if (!ptx::mbar_wait(&bar_p_ready[b], ph, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                if (!wait_part(kPartDomn, it)) { ok = false; break; }
                const uint32_t dmn = ptx::smem_addr(PP ? pp_addr(kPartDomn, it) : st_domn(s));
#pragma unroll
                for (int kk = 0; kk < W / G::kKStep; ++kk)
                    ptx::mma_tf32_ts(tmem + Cfg::kColDVkv, tmem + Cfg::kColS + b * W + kk * G::kKStep, desc_mnmajor<G>(dmn, kk, W), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                release_part(kPartDomn, it);
                if (it + NG < n_it && !issue_s(it + NG)) { ok = false; break; }
                // dK_j += dS^T Q_i   (Eq. 19 without the scale); dS^T from the dP^T columns.
                if (!ptx::mbar_wait(&bar_ds_ready[b], ph, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                if (!wait_part(kPartQmn, it)) { ok = false; break; }
                const uint32_t qmn = ptx::smem_addr(PP ? pp_addr(kPartQmn, it) : st_qmn(s));
#pragma unroll
                for (int kk = 0; kk < W / G::kKStep; ++kk)
                    ptx::mma_tf32_ts(tmem + Cfg::kColDKkv, tmem + Cfg::kColDPkv + b * W + kk * G::kKStep, desc_mnmajor<G>(qmn, kk, W), idesc_kv, (it > 0 || kk > 0) ? 1u : 0u);
                if constexpr (PP) release_part(kPartQmn, it);
                else ptx::mma_commit(&bar_empty[s]);
                if (it + NG < n_it && !issue_dp(it + NG)) { ok = false; break; }
            }
            if (ok) {
                ptx::mma_commit(&bar_dkv_full);
            } else {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else {
        // ------------------------------------------------ P / dS warpgroup(s)
        const int grp = (warp - 2) >> 2;                 // takes sub-tiles it = grp (mod NG)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // key row inside the tile
        const bool key_valid = kv_row0 + r < p.Nk;
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        bool ok = true;
        if constexpr (KT) {
            // K row r (TF32-rounded copy) into tensor memory; zeros past Nk (group 0).
            if (n_it > 0 && grp == 0) {
                const float4* krow = reinterpret_cast<const float4*>(
                    p.k32 + (static_cast<size_t>(bh) * p.Nk + (key_valid ? kv_row0 + r : 0)) * D);
#pragma unroll
                for (int c0 = 0; c0 < D; c0 += 32) {
                    uint32_t u[32];
#pragma unroll
                    for (int q4 = 0; q4 < 8; ++q4) {
                        const float4 x = key_valid ? __ldg(krow + c0 / 4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
                        u[4 * q4 + 0] = __float_as_uint(x.x);
                        u[4 * q4 + 1] = __float_as_uint(x.y);
                        u[4 * q4 + 2] = __float_as_uint(x.z);
                        u[4 * q4 + 3] = __float_as_uint(x.w);
                    }
                    ptx::tmem_st32(lane_base + Cfg::kColKT + c0, u);
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_kt_ready);
            }
        }
        const uint32_t col_s = Cfg::kColS + grp * W, col_dp = Cfg::kColDPkv + grp * W;
        for (int it = grp; it < n_it; it += NG) {
            const uint32_t ph = static_cast<uint32_t>(it / NG) & 1u;
            const int q0 = q_row_of(it);
            const size_t qv = static_cast<size_t>(q_head_of(it)) * p.n_pad + q0;
            const float* l2q = p.l2 + qv;
            const float* dvq = p.dvec + qv;
            // Some query of this sub-tile precedes some key of the tile.
            const bool mask = p.causal && q0 < kv_row0 + kTileRows - 1;
            // ---- P^T = exp2(S^T * scale*log2(e) - L*log2(e))   (Eq. 14), in place
            if (!ptx::mbar_wait(&bar_s_full[grp], ph, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pu[W];
            tmem_ld_cols<W>(lane_base + col_s, pu);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < W; c += 4) {
                const float4 lv = __ldg(reinterpret_cast<const float4*>(l2q + c));
                const float lq[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    float pe = ptx::ex2_approx(fmaf(__uint_as_float(pu[c + h]), sl2, -lq[h]));
                    if ((mask && q0 + c + h < kv_row0 + r) || !key_valid) pe = 0.f;
                    pu[c + h] = __float_as_uint(pe);
                }
            }
            bwd32_store_p<W>(lane_base + col_s, pu);
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_p_ready[grp]);
            // ---- dS^T = P^T o (dP^T - D)   (Eq. 17), in place over dP^T
            if (!ptx::mbar_wait(&bar_dp_full[grp], ph, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            bwd32_ds_inplace<W>(lane_base + col_dp, pu, [&](int c) { return __ldg(dvq + c); });
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_ds_ready[grp]);
        }
        // ---------------- epilogue (group 0): dV -> sV, dK * scale -> sK, then TMA stores.
        if (grp == 0) {
        if (ok && n_it > 0) ok = ptx::mbar_wait(&bar_dkv_full, 0, &abort_flag, tmo);
        if (ok) {
            ptx::tc_fence_after();
            bwd32_stage_rows<G>(lane_base + Cfg::kColDVkv, r, 1.f, sV, n_it == 0);
            bwd32_stage_rows<G>(lane_base + Cfg::kColDKkv, r, p.scale, sDK, n_it == 0);
            ptx::fence_async_smem();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok && threadIdx.x == 64) {
            for (int bx = 0; bx < G::kNBoxK; ++bx) {
                ptx::tma_store_3d(&tm_dv, sV + bx * kTileRows * G::kRowBK, bx * G::kBoxK, kv_row0, bh);
                ptx::tma_store_3d(&tm_dk, sDK + bx * kTileRows * G::kRowBK, bx * G::kBoxK, kv_row0, bh);
            }
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

// ------------------------------------------------------------------ dQ pass

// One CTA per (query tile i, head); Q_i and dO_i stay resident, the key rows
// query tile i sees stream through in sub-tiles of W rows.  Per sub-tile the
// MMA issuer runs S = Q K^T, dP = dO V^T, dQ += dS K, issuing the next S as
// soon as the warpgroup has read this one and the next dP right after dQ.
// With a block mask (SPARSE) only the sub-tiles of key tiles whose block with
// query tile i is set are visited, found by each thread walking the mask row.
template <int D, bool SPARSE = false>
__global__ void __launch_bounds__(Bwd32Cfg<D>::kThreadsQ, 1)
fa2_bwd32_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_kk, const __grid_constant__ CUtensorMap tm_kmn,
                    const __grid_constant__ CUtensorMap tm_vk, const __grid_constant__ CUtensorMap tm_dq,
                    const BwdParams p) {
    // Programmatic dependent launch: the next kernel may be scheduled now; wait for
    // the previous kernel of the stream before touching global memory.
    ptx::pdl_launch_dependents();
    ptx::pdl_wait();
    using Cfg = Bwd32Cfg<D>;
    using G = typename Cfg::G;
    constexpr int W = Cfg::kWq;
    constexpr int ST = Cfg::kStQ;
    constexpr int TK = Cfg::tile_k(kTileRows);
    constexpr int SK = Cfg::tile_k(W);
    constexpr int SB = Cfg::q_stage(W);

    extern __shared__ uint8_t smem_raw[];
    constexpr int NG = Cfg::kGroupsQ;                   // P / dS warpgroups (S, dP buffers)
    static_assert(NG == 1 || NG * W <= 128, "S / dP buffers exceed their TMEM columns");
    __shared__ uint64_t bar_qdo_full, bar_full[ST], bar_empty[ST];
    __shared__ uint64_t bar_s_full[NG], bar_dp_full[NG], bar_s_read[NG], bar_ds_ready[NG], bar_dq_done, bar_drain;
    __shared__ uint64_t bar_qt_ready;                   // Q and dO written to tensor memory (QT)
    __shared__ uint32_t tmem_slot;
    __shared__ volatile uint32_t abort_flag;
    __shared__ int s_cnt;                               // block-sparse: key sub-tiles

    const uint32_t raw = ptx::smem_addr(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    constexpr bool QT = Cfg::kQInTmem;
    uint8_t* sQ = smem;                                 // unused when Q, dO are in tensor memory
    uint8_t* sDO = sQ + TK;
    uint8_t* sStage = QT ? smem : sDO + TK;
    // dQ is staged for its store where Q was, or in the (then idle) first stage.
    uint8_t* sDQ = QT ? sStage : sQ;
    // Stage s: K (K-major) | V (K-major) | K (MN-major).
    auto st_kk = [&](int s) { return sStage + s * SB; };
    auto st_vk = [&](int s) { return sStage + s * SB + SK; };
    auto st_kmn = [&](int s) { return sStage + s * SB + 2 * SK; };

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Work item: causal query tile i sees keys < 128 (i + 1); longest first.
    const int item = blockIdx.x;
    const int rank = item / p.BH;
    const int bh = item - rank * p.BH;
    const int q_tile = p.causal ? (p.n_tiles - 1 - rank) : rank;
    const int q_row0 = q_tile * kTileRows;
    const int n_sub = (p.Nk + W - 1) / W;               // key sub-tiles
    const int lim = (q_row0 + kTileRows) / W;
    const int bh_kv = kv_head_of(bh, p.H, p.H_kv, p.group);
    constexpr int R = kTileRows / W;                    // sub-tiles per 128-row tile
    // Block-sparse: key tiles t < n_lim whose block with this query tile is set.
    const int n_lim = p.causal ? min(q_tile + 1, p.n_tiles_k) : p.n_tiles_k;
    const uint8_t* mask_row = SPARSE ? p.block_mask + static_cast<size_t>(q_tile) * p.n_tiles_k : nullptr;
    auto blk_set = [&](int t) { return __ldg(mask_row + t) != 0; };
    if (SPARSE && warp == 0) {
        int c = 0;
        for (int base = 0; base < n_lim; base += 32)
            c += __popc(__ballot_sync(0xffffffffu, base + lane < n_lim && blk_set(base + lane)));
        // R sub-tiles per set key tile; the last key tile's end at n_sub.
        const bool last = n_lim == p.n_tiles_k && n_lim > 0 && blk_set(n_lim - 1);
        if (lane == 0) s_cnt = c * R - (last ? p.n_tiles_k * R - n_sub : 0);
    }
    MaskWalk walker;
    // Key sub-tile of step j.
    auto kvs_of = [&](int j) { return SPARSE ? walker.at(j / R, n_lim, blk_set) * R + j % R : j; };

    if (threadIdx.x == 0) {
        abort_flag = 0u;
        ptx::mbar_init(&bar_qdo_full, 1);
        for (int s = 0; s < ST; ++s) {
            ptx::mbar_init(&bar_full[s], 1);
            ptx::mbar_init(&bar_empty[s], 1);
        }
        for (int b = 0; b < NG; ++b) {
            ptx::mbar_init(&bar_s_full[b], 1);
            ptx::mbar_init(&bar_dp_full[b], 1);
            ptx::mbar_init(&bar_s_read[b], 4);
            ptx::mbar_init(&bar_ds_ready[b], 4);
        }
        ptx::mbar_init(&bar_dq_done, 1);
        ptx::mbar_init(&bar_drain, 1);
        ptx::mbar_init(&bar_qt_ready, 4);
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
    // Key sub-tile steps; none for an empty block row, whose dQ is written as 0.
    const int n_kv = SPARSE ? s_cnt : (p.causal ? (lim < n_sub ? lim : n_sub) : n_sub);

    if (warp == 0) {
        // ------------------------------------------------ TMA producer
        if (lane == 0 && n_kv > 0) {
            ptx::prefetch_tmap(&tm_kk);
            ptx::prefetch_tmap(&tm_kmn);
            ptx::prefetch_tmap(&tm_vk);
            const uint64_t keep = ptx::policy_evict_last();
            if (!QT) {
                ptx::mbar_arrive_expect_tx(&bar_qdo_full, 2 * TK);
                for (int b = 0; b < G::kNBoxK; ++b) {
                    ptx::tma_load_3d(sQ + b * kTileRows * G::kRowBK, &tm_q, &bar_qdo_full, b * G::kBoxK, q_row0, bh);
                    ptx::tma_load_3d(sDO + b * kTileRows * G::kRowBK, &tm_do, &bar_qdo_full, b * G::kBoxK, q_row0, bh);
                }
            }
            int issued = 0;
            for (int j = 0; j < n_kv; ++j) {
                const int s = j % ST;
                if (j >= ST && !ptx::mbar_wait(&bar_empty[s], ((j / ST) & 1) ^ 1, &abort_flag, tmo)) break;
                const int row0 = kvs_of(j) * W;
                ptx::mbar_arrive_expect_tx(&bar_full[s], SB);
                for (int b = 0; b < G::kNBoxK; ++b) {
                    ptx::tma_load_3d_hint(st_kk(s) + b * W * G::kRowBK, &tm_kk, &bar_full[s], b * G::kBoxK, row0, bh_kv, keep);
                    ptx::tma_load_3d_hint(st_vk(s) + b * W * G::kRowBK, &tm_vk, &bar_full[s], b * G::kBoxK, row0, bh_kv, keep);
                }
                for (int b = 0; b < G::kNBoxMN; ++b)
                    ptx::tma_load_3d_hint(st_kmn(s) + b * W * G::kRowBMN, &tm_kmn, &bar_full[s], b * G::kBoxMN, row0, bh_kv, keep);
                issued = j + 1;
            }
            if (abort_flag) {
                constexpr uint64_t kDrainNs = 20000000ull;
                if (!QT) ptx::mbar_wait_drain(&bar_qdo_full, 0, kDrainNs);
                for (int t = issued - 1; t >= 0 && t >= issued - ST; --t)
                    ptx::mbar_wait_drain(&bar_full[t % ST], (t / ST) & 1, kDrainNs);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0 && n_kv > 0) {
            constexpr uint32_t idesc_s = ptx::instr_desc(G::kFmt, 128, W, false, false);
            constexpr uint32_t idesc_dq = ptx::instr_desc(G::kFmt, 128, G::kNOut, false, true);
            const uint32_t q_addr = ptx::smem_addr(sQ);
            const uint32_t do_addr = ptx::smem_addr(sDO);
            // S = Q_i K_j^T   (Eq. 13)
            auto issue_s = [&](int j) -> bool {
                const int s = j % ST;
                if (!ptx::mbar_wait(&bar_full[s], (j / ST) & 1, &abort_flag, tmo)) return false;
                ptx::tc_fence_after();
                const uint32_t ka = ptx::smem_addr(st_kk(s));
                const int b = j % NG;
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk) {
                    if constexpr (QT)
                        ptx::mma_tf32_ts(tmem + Cfg::kColS + b * W, tmem + Cfg::kColQT + kk * G::kKStep, desc_kmajor<G>(ka, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_tf32_ss(tmem + Cfg::kColS + b * W, desc_kmajor<G>(q_addr, kk), desc_kmajor<G>(ka, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bar_s_full[b]);
                return true;
            };
            // dP = dO_i V_j^T   (Eq. 16); the stage is already full.
            auto issue_dp = [&](int j) {
                const uint32_t va = ptx::smem_addr(st_vk(j % ST));
                const int b = j % NG;
#pragma unroll
                for (int kk = 0; kk < G::kStepsD; ++kk) {
                    if constexpr (QT)
                        ptx::mma_tf32_ts(tmem + Cfg::kColDPq + b * W, tmem + Cfg::kColDOT + kk * G::kKStep, desc_kmajor<G>(va, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                    else
                        ptx::mma_tf32_ss(tmem + Cfg::kColDP + b * W, desc_kmajor<G>(do_addr, kk), desc_kmajor<G>(va, kk, W), idesc_s, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(&bar_dp_full[b]);
            };
            bool ok = QT ? ptx::mbar_wait(&bar_qt_ready, 0, &abort_flag, tmo)
                         : ptx::mbar_wait(&bar_qdo_full, 0, &abort_flag, tmo);
            for (int i = 0; ok && i < NG && i < n_kv; ++i) {
                ok = issue_s(i);
                if (ok) issue_dp(i);
            }
            // Sub-tile j + NG reuses the buffers of sub-tile j: its S once the
            // warpgroup has read S(j), its dP after dQ(j).
            for (int j = 0; ok && j < n_kv; ++j) {
                const int b = j % NG;
                const uint32_t ph = static_cast<uint32_t>(j / NG) & 1u;
                if (j + NG < n_kv) {
                    if (!ptx::mbar_wait(&bar_s_read[b], ph, &abort_flag, tmo)) { ok = false; break; }
                    if (!issue_s(j + NG)) { ok = false; break; }
                }
                // dQ_i += dS K_j   (Eq. 18 without the scale); dS from the dP columns.
                if (!ptx::mbar_wait(&bar_ds_ready[b], ph, &abort_flag, tmo)) { ok = false; break; }
                ptx::tc_fence_after();
                const uint32_t kmn = ptx::smem_addr(st_kmn(j % ST));
#pragma unroll
                for (int kk = 0; kk < W / G::kKStep; ++kk)
                    ptx::mma_tf32_ts(tmem + Cfg::kColDQq, tmem + Cfg::kColDPq + b * W + kk * G::kKStep, desc_mnmajor<G>(kmn, kk, W), idesc_dq, (j > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(&bar_empty[j % ST]);
                if (j + NG < n_kv) issue_dp(j + NG);
            }
            if (ok) {
                ptx::mma_commit(&bar_dq_done);
            } else {
                ptx::mma_commit(&bar_drain);
                ptx::mbar_wait_drain(&bar_drain, 0, 20000000ull);
            }
        }
    } else {
        // ------------------------------------------------ P / dS warpgroup(s)
        const int grp = (warp - 2) >> 2;                 // takes sub-tiles j = grp (mod NG)
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;               // query row inside the tile
        const uint32_t lane_base = tmem + ptx::tmem_lane_offset(quarter * 32);
        const float sl2 = p.scale_log2;
        const size_t vrow = static_cast<size_t>(bh) * p.n_pad + q_row0 + r;
        const float l2r = p.l2[vrow];                    // L_i * log2(e) (+inf past N)
        const float dr = p.dvec[vrow];                   // D_i (0 past N)
        bool ok = true;
        if constexpr (QT) {
            // Q and dO row r (TF32-rounded copies) into tensor memory; zeros past N
            // (group 0).
            if (n_kv > 0 && grp == 0) {
                const bool row_valid = q_row0 + r < p.N;
                const size_t row_off = (static_cast<size_t>(bh) * p.N + (row_valid ? q_row0 + r : 0)) * D;
#pragma unroll
                for (int t = 0; t < 2; ++t) {
                    const float4* src = reinterpret_cast<const float4*>((t == 0 ? p.q32 : p.do32) + row_off);
                    const uint32_t col = t == 0 ? Cfg::kColQT : Cfg::kColDOT;
#pragma unroll
                    for (int c0 = 0; c0 < D; c0 += 32) {
                        uint32_t u[32];
#pragma unroll
                        for (int q4 = 0; q4 < 8; ++q4) {
                            const float4 x = row_valid ? __ldg(src + c0 / 4 + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
                            u[4 * q4 + 0] = __float_as_uint(x.x);
                            u[4 * q4 + 1] = __float_as_uint(x.y);
                            u[4 * q4 + 2] = __float_as_uint(x.z);
                            u[4 * q4 + 3] = __float_as_uint(x.w);
                        }
                        ptx::tmem_st32(lane_base + col + c0, u);
                    }
                }
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&bar_qt_ready);
            }
        }
        const uint32_t col_s = Cfg::kColS + grp * W, col_dp = Cfg::kColDPq + grp * W;
        for (int j = grp; j < n_kv; j += NG) {
            const uint32_t ph = static_cast<uint32_t>(j / NG) & 1u;
            const int k0 = kvs_of(j) * W;
            const bool mask = p.causal && k0 + W - 1 > q_row0;   // some key follows some query
            const int kv_valid = p.Nk - k0;                         // key columns < Nk
            // ---- P = exp2(S * scale*log2(e) - L*log2(e))   (Eq. 14), kept in registers
            if (!ptx::mbar_wait(&bar_s_full[grp], ph, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            uint32_t pu[W];
            tmem_ld_cols<W>(lane_base + col_s, pu);
            ptx::tmem_wait_ld();
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_s_read[grp]);
#pragma unroll
            for (int c = 0; c < W; ++c) {
                float pe = ptx::ex2_approx(fmaf(__uint_as_float(pu[c]), sl2, -l2r));
                if ((mask && k0 + c > q_row0 + r) || c >= kv_valid) pe = 0.f;
                pu[c] = __float_as_uint(pe);
            }
            // ---- dS = P o (dP - D)   (Eq. 17) -> TMEM over dP
            if (!ptx::mbar_wait(&bar_dp_full[grp], ph, &abort_flag, tmo)) { ok = false; break; }
            ptx::tc_fence_after();
            bwd32_ds_inplace<W>(lane_base + col_dp, pu, [&](int) { return dr; });
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(&bar_ds_ready[grp]);
        }
        // ---------------- epilogue (group 0): dQ * scale -> sQ -> TMA store (zeros
        // when no key tile was visited; nothing was loaded into sQ then).
        if (grp == 0) {
        if (ok && n_kv > 0) ok = ptx::mbar_wait(&bar_dq_done, 0, &abort_flag, tmo);
        if (ok) {
            ptx::tc_fence_after();
            bwd32_stage_rows<G>(lane_base + Cfg::kColDQq, r, p.scale, sDQ, n_kv == 0);
            ptx::fence_async_smem();
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (ok && threadIdx.x == 64) {
            for (int bx = 0; bx < G::kNBoxK; ++bx)
                ptx::tma_store_3d(&tm_dq, sDQ + bx * kTileRows * G::kRowBK, bx * G::kBoxK, q_row0, bh);
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
