// Shared definitions of the GDN kernels: status word, problem description, smem layout
// constants.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace gdn {

// Device status word: 0 = OK, otherwise the first error a kernel recorded (the C-ABI status
// codes; GDN_ERR_TIMEOUT when a bounded wait ran out). Read and cleared by gdn_sync_status.
__device__ int g_status;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_status, 0, code); }

constexpr int kErrTimeout = 6;  // == GDN_ERR_TIMEOUT

// The (cos, sin) table of the 3D RoPE (see rope_kernel.cuh for the reading) and its layout. The
// head dimension's D/2 pairs j split into the time slice [0, pt), the grid-row slice
// [pt, pt + ph) and the grid-column slice [pt + ph, pt + 2 ph). For each axis and each position
// on it (frame, grid row, grid column) the table holds one row of len entries indexed by the
// absolute pair index: pair j at row offset j - j0, j0 = the axis's first pair rounded down to
// even, len even, entries of the row outside the axis's slice (1, 0). Every row starts at an
// even entry, so pairs (j, j + 1) with j even are one aligned 16-byte load from either pair's
// axis. Rows: frame t at t * len_t, grid row r at off_h + r * len_h, grid column c at
// off_w + c * len_w.
struct RopeArgs {
  const float2* tab = nullptr;
  int grid_h = 1, grid_w = 1;
  int pt = 0, ph = 0;                   // pairs of the time slice and of the row (= column) slice
  int len_t = 0, len_h = 0, len_w = 0;  // row lengths of the three axes (even)
  int j0_h = 0, j0_w = 0;               // first pair of the row / column slice, rounded down to even
  int off_h = 0, off_w = 0;             // first table entries of the row and column axes
  int n_rc = 0;  // entries of the grid-row and grid-column rows (from off_h to the table's end)
};

// One problem: q/k/v/out are [B, T, N, H, D] bf16, gamma/beta [B, T, H] f32.
struct Problem {
  int B, H, T, N, D;
  float key_scale;
  // fp8 (e4m3) inputs: per (b, t, h) scales [B, T, H] f32, q = q8 * q_scale etc.; unused for bf16
  const float* q_scale = nullptr;
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
  // 3D RoPE of q and k (forward with the rotary prologue only)
  RopeArgs rope;
};

// Hand-off state of the fused forward, in device memory and zeroed before each call. One
// persistent grid runs three roles: stats CTAs write A_t, B_t into per-head rings of R slots,
// chain CTAs consume them and write S_t into per-head rings of Rs slots, output CTAs consume S_t.
struct Handoff {
  int* stats_flag;  // [B*H*T] 1 once A_t, B_t of (bh, t) are in ring slot t % R
  int* out_flag;    // [B*H*T] 1 once the output of (bh, t) has loaded S_t (its slot is free)
  int* chain_prog;  // [B*H]   number of frames whose S_t the chain has stored
  int* abort;       // set by the first CTA that gives up a wait; every wait then returns
  int* next_item;   // this role's work counter (stats and output roles take items dynamically)
  int R;            // A_t / B_t ring slots per head (how far the statistics may run ahead)
  int Rs;           // S_t ring slots per head (how far the outputs may lag behind)
  int withhold;     // test hook: frame whose statistics of head 0 are never published (-1: none)
  int base;         // first blockIdx.x of this role
  int count;        // CTAs in this role
  // outputs in publish order: the chain appends item t*B*H + bh (+1) at ready_items[ready_tail++]
  // as soon as S_t is visible, and output CTAs take queue positions from next_item, so an output
  // CTA only waits when no published state is left anywhere (not on one lagging head). A fixed
  // frame-major order, which would let an output CTA load its Q tiles before the chain reaches
  // its frame, measured slower on the 480p and 720p clips.
  int* ready_items = nullptr;  // [B*H*T], 0 = not yet written
  int* ready_tail = nullptr;
};

// Dynamic work distribution inside a CTA of the fused forward: the producer thread takes the
// next item of its role from a global counter (so items start in global frame-major order,
// whichever CTA is free) and passes the item id to the CTA's other warps through an 8-slot ring
// of (id, mbarrier) pairs. The producer runs at most a few items ahead of the last consumer
// (its tile stages and the two TMEM accumulators bound it), so 8 slots are never overrun.
struct ItemRing {
  int* ids;        // shared [8]
  uint64_t* bars;  // shared [8], arrival count 1
  __device__ __forceinline__ long produce(int li, int* counter, long n_items) {
    long it = atomicAdd(counter, 1);
    if (it >= n_items) it = -1;
    ids[li & 7] = static_cast<int>(it);
    mbar_arrive(&bars[li & 7]);
    return it;
  }
  // Same, with the item taken from a queue of published items: queue position from the counter,
  // then (bounded) wait until that position is written. -2 if the wait ran out.
  __device__ __forceinline__ long produce_queued(int li, int* counter, const int* queue,
                                                 long n_items, const int* abort) {
    const long pos = atomicAdd(counter, 1);
    long it = -1;
    if (pos < n_items) it = wait_flag_ge(queue + pos, 1, abort) ? ld_acquire(queue + pos) - 1 : -2;
    ids[li & 7] = static_cast<int>(it);
    mbar_arrive(&bars[li & 7]);
    return it;
  }
  // -2 if the wait timed out, -1 once the role's items are exhausted
  __device__ __forceinline__ long consume(int li) {
    if (!mbar_wait(&bars[li & 7], (li >> 3) & 1)) return -2;
    return ids[li & 7];
  }
};

__device__ __forceinline__ void give_up(const Handoff& hf, volatile int* local_abort) {
  record_error(kErrTimeout);
  if (hf.abort != nullptr) atomicExch(hf.abort, 1);
  *local_abort = 1;
}

// B_t storage used between the statistics and the chain: element (v, k) of the D x D matrix at
// float index ((k / 4) * D + v) * 4 + k % 4, i.e. 16-byte groups of four keys, consecutive value
// rows adjacent. A warp handling 32 consecutive rows then reads or writes 512 contiguous bytes per
// group, for both the writer (one thread per row) and the reader (one thread per row).
__host__ __device__ __forceinline__ long b4_index(int v, int k, int D) {
  return (static_cast<long>(k >> 2) * D + v) * 4 + (k & 3);
}

// S_t storage between the chain and the output GEMM: a DP x DP bf16 matrix (zero-padded past D)
// as K-major 8 x 16-byte core matrices, element (v, k) at bf16 index ((k / 8) * DP + v) * 8 +
// k % 8. It is directly a no-swizzle MMA operand (LBO = DP*16 bytes between key groups, SBO =
// 128 bytes between 8-row groups), one contiguous DP*DP*2-byte block per frame, and a warp that
// owns 32 consecutive rows writes it as 512 contiguous bytes per key group.
__host__ __device__ __forceinline__ long s8_offset_bytes(int v, int k, int DP) {
  return (static_cast<long>(k >> 3) * DP + v) * 16 + (k & 7) * 2;
}

// Record of one chunk's composed frame maps in the chunked forward (S_end = S_start * P + C):
// P transposed as two DP x DP bf16 matrices in the layout of s8_offset_bytes (the bf16 value
// of P, then the bf16 value of the remainder P - hi), followed by C as D x D f32 in the layout of
// b4_index. 128 KB at DP = 128.
__host__ __device__ constexpr long chunk_map_bytes(int DP) {
  return 2L * DP * DP * 2 + static_cast<long>(DP) * DP * 4;
}

// Start state of one chunk in the chunked forward: D x D f32 in the four-key interleaved layout
// of b4_index (the scan's epilogue warps store and the replay's read 512 contiguous bytes per
// warp and key group). Sized for DP so records stay 256-byte aligned.
__host__ __device__ constexpr long chunk_start_bytes(int DP) { return static_cast<long>(DP) * DP * 4; }

// TMA box: 64 bf16 (128 B, one swizzle row) x 128 rows.
constexpr int kRowsPerTile = 128;
constexpr int kBoxBytes = 128 * 128;  // 16 KB

// Round an address up to 1 KB (swizzle-atom alignment of every tile).
__device__ __forceinline__ uint8_t* align1k(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace gdn
