// fa2_traits.cuh -- compile-time tile geometry shared by the forward and
// backward kernels, and the shared-memory tile layouts the tensor memory
// accelerator (TMA) writes and the tcgen05 MMA reads.
//
// A "tile" is 128 consecutive rows (queries or keys) of one head, all d
// columns.  The handout does not tile the head dimension (CS336 A2 Systems
// handout section 4.2.2: "we will not tile along the hidden dimension d"), and
// neither do we: a tile is staged in shared memory as NBOX boxes of BOX
// columns each (one TMA copy per box), BOX chosen so that one box row is the
// width of a hardware swizzle pattern.
//
// Two staging geometries exist for the same tensor:
//   K-major  - the operand's contraction dimension runs along d (Q and K in
//              S = Q K^T).  Rows are ROWB = BOX*ES bytes, swizzled with the
//              32/64/128-byte pattern of that width.
//   MN-major - the contraction runs along the 128 rows and d is the output
//              dimension (V in O += P V).  16-bit types reuse the K-major
//              staging.  32-bit (TF32) operands must use 128-byte rows with
//              32-byte swizzle atoms, whose 8-row groups are 512 bytes apart.
#pragma once

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fa2 {

constexpr int kTileRows = 128;  // B_q = B_k = 128 rows per tile

// Grouped-query attention: query heads h = g * group .. g * group + group - 1
// of a batch share key/value head g.  `bh` indexes [B * H] query heads; the
// result indexes [B * H_kv] key/value heads (H_kv = H / group; group = 1 is
// plain multi-head attention).
__host__ __device__ inline int kv_head_of(int bh, int H, int H_kv, int group) {
    return (bh / H) * H_kv + (bh % H) / group;
}

// Work items of a (rank, head) grid in groups of `hg` heads: the items of a
// group cover its heads at every rank, rank-major inside the group, so the CTAs
// resident together read the K/V (or Q/dO) of few heads, which stay in L2;
// inside a group the lowest rank (the longest item under the causal rule, as
// the callers number ranks) comes first.  hg >= n_heads is the plain rank-major
// order.
__host__ __device__ inline void grouped_item(int item, int n_rank, int n_heads, int hg, int& rank, int& head) {
    const int per_group = hg * n_rank;
    const int g = item / per_group;
    const int in_group = item - g * per_group;
    const int heads_here = (n_heads - g * hg) < hg ? (n_heads - g * hg) : hg;
    rank = in_group / heads_here;
    head = g * hg + (in_group - rank * heads_here);
}

// Heads per group for grouped_item: groups of about 600 items (four waves of
// 148 SMs), the heads split evenly over the groups.
inline int heads_per_group(int n_heads, int n_rank) {
    const long long items = static_cast<long long>(n_heads) * n_rank;
    const int groups = static_cast<int>((items + 599) / 600);
    return groups <= 1 ? n_heads : (n_heads + groups - 1) / groups;
}

// Block-sparse attention ("Notes on flashattention", section "Block-sparse
// Flashattention"): a byte per (query tile, key tile) pair of kTileRows x
// kTileRows blocks, row-major with one row per query tile; zero blocks are
// skipped.  A CTA compacts the tiles it visits into a shared-memory list of
// kMaxMaskTiles 16-bit entries; a CTA whose tiles do not fit there (more steps,
// or tile indices wider than the entries) walks the mask itself (MaskWalk).
constexpr int kMaxMaskTiles = 512;

// Warp-cooperative compaction (whole warp): writes, in increasing order, the
// value val(t) of every t in [0, n) with keep(t) into list[] (the first
// kMaxMaskTiles of them), and returns the count of all of them (the same in
// every lane).
template <class Keep, class Val>
__device__ __forceinline__ int warp_compact(uint16_t* list, int n, Keep keep, Val val) {
    const int lane = threadIdx.x & 31;
    int count = 0;
    for (int base = 0; base < n; base += 32) {
        const int t = base + lane;
        const bool k = t < n && keep(t);
        const unsigned bal = __ballot_sync(0xffffffffu, k);
        if (k && count + __popc(bal & ((1u << lane) - 1u)) < kMaxMaskTiles)
            list[count + __popc(bal & ((1u << lane) - 1u))] = static_cast<uint16_t>(val(t));
        count += __popc(bal);
    }
    return count;
}

// The s-th (s = 0, 1, 2, ...) index t in [0, n) with keep(t), found by walking
// the mask from the previous answer: one thread's replacement for the
// shared-memory list.  Steps are asked for in increasing order (asking for an
// earlier step restarts the walk); a step past the last index gives n.
struct MaskWalk {
    int step = -1;   // step number of `pos`
    int pos = -1;    // index of that step
    template <class Keep>
    __device__ __forceinline__ int at(int s, int n, Keep keep) {
        if (s < step) { step = -1; pos = -1; }
        while (step < s && pos < n) {
            ++pos;
            while (pos < n && !keep(pos)) ++pos;
            ++step;
        }
        return pos < n ? pos : n;
    }
};

// Device status codes the kernels record (same values as fa2_status).
constexpr uint32_t kDevStatusTimeout = 8;

// ES = element bytes (2 or 4); for 2-byte inputs F16 selects fp16 over bf16.
template <int ES, int D, bool F16 = false>
struct TileGeom {
    static_assert(!(F16 && ES != 2), "fp16 inputs are 2-byte elements");
    static constexpr int kES = ES;
    static constexpr int kD = D;
    static constexpr bool kF32 = (ES == 4);
    static constexpr bool kF16 = F16;
    // K-major staging.
    static constexpr int kBoxK = (D * ES >= 128) ? (128 / ES) : D;
    static constexpr int kRowBK = kBoxK * ES;
    static constexpr int kNBoxK = (D + kBoxK - 1) / kBoxK;
    static constexpr int kTileBytesK = kNBoxK * kTileRows * kRowBK;
    static constexpr uint32_t kLayoutK = ptx::layout_for_row_bytes(kRowBK);
    // MN-major staging.
    static constexpr int kBoxMN = kF32 ? 32 : kBoxK;
    static constexpr int kRowBMN = kBoxMN * ES;
    static constexpr int kNBoxMN = (D + kBoxMN - 1) / kBoxMN;
    static constexpr int kTileBytesMN = kNBoxMN * kTileRows * kRowBMN;
    static constexpr uint32_t kLayoutMN = kF32 ? 1u : kLayoutK;
    static constexpr uint32_t kSboMN = kF32 ? 512u : 8u * kRowBMN;
    // MMA shape facts.
    static constexpr int kKStep = 32 / ES;                        // K per MMA instruction
    static constexpr int kStepsD = (D + kKStep - 1) / kKStep;    // MMAs to contract over d
    static constexpr int kStepsRows = kTileRows / kKStep;        // MMAs to contract over 128 rows
    static constexpr int kNOut = (D + 15) / 16 * 16;              // MMA N when d is the output dim
    static constexpr uint32_t kFmt = kF32 ? ptx::kFmtTF32 : (F16 ? ptx::kFmtF16 : ptx::kFmtBF16);
    // Two fp32 values rounded (nearest even) to the 16-bit input type, packed
    // with the first in the low half; and the reverse, exact.
    static __device__ __forceinline__ uint32_t pack2(float lo, float hi) {
        if constexpr (F16) return ptx::pack_f16x2(lo, hi);
        else return ptx::pack_bf16x2(lo, hi);
    }
    static __device__ __forceinline__ void unpack2(uint32_t w, float& lo, float& hi) {
        if constexpr (F16) ptx::unpack_f16x2(w, lo, hi);
        else ptx::unpack_bf16x2(w, lo, hi);
    }
    static constexpr int kPCols = kF32 ? 128 : 64;                // TMEM columns of a 128-wide P row
};

// Descriptor of the k-th contraction step of a K-major staged tile whose
// boxes each hold `rows` rows.
template <class G>
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile_addr, int k, int rows = kTileRows) {
    const int off = k * 32;  // 32 bytes of K per MMA instruction
    const uint32_t a = tile_addr + (off / G::kRowBK) * rows * G::kRowBK + (off % G::kRowBK);
    return ptx::smem_desc(a, 16, 8 * G::kRowBK, G::kLayoutK);
}

// Descriptor of the k-th contraction step (k-th group of kKStep rows) of an
// MN-major staged tile whose boxes each hold `rows` rows.
template <class G>
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile_addr, int k, int rows = kTileRows) {
    const uint32_t a = tile_addr + k * G::kKStep * G::kRowBMN;
    return ptx::smem_desc(a, rows * G::kRowBMN, G::kSboMN, G::kLayoutMN);
}

// Byte offset, inside a K-major staged tile, of the 16-byte chunk holding
// columns [col, col + 16/ES) of `row` (col a multiple of 16/ES).  Applies the
// swizzle the TMA uses for rows of kRowBK bytes (16-byte chunk index XOR the
// row's position inside the 1024/512/256-byte swizzle period).
template <class G>
__device__ __forceinline__ uint32_t kmajor_chunk_offset(int row, int col) {
    const int box = col / G::kBoxK;
    const int chunk = (col % G::kBoxK) * G::kES / 16;
    constexpr int kChunks = G::kRowBK / 16;
    const int sw = ((row * G::kRowBK) >> 7) & (kChunks - 1);
    return box * kTileRows * G::kRowBK + row * G::kRowBK + ((chunk ^ sw) * 16);
}

}  // namespace fa2
