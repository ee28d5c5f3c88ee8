// common.cuh -- constants and small device helpers shared by the plan, forward
// and backward kernels of the sigmoid-attention library.
#pragma once

#include <algorithm>
#include <cstdint>
#include <type_traits>
#include <utility>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sigattn {

// Rows of one work item, per call kind. A work item is one block of
// consecutive rows of one (batch, head) slice holding >= 1 valid token:
//  * forward: 256 query rows (two 128-row query tiles sharing each K/V block),
//  * dQ:      128 query rows,
//  * dK/dV:   128 key rows.
// Every inner loop walks blocks of columns (keys for forward/dQ, queries for
// dK/dV; 128 wide, 64 for dK/dV at d = 128) only up to the last block holding
// a valid token, so fully padded blocks are never touched on either side.
enum Kind : int { kKindFwd = 0, kKindDq = 1, kKindDkdv = 2 };
constexpr int kFwdItemRows = 256;
constexpr int kBwdItemRows = 128;
constexpr int kColBlock = 128;
constexpr int kMaxBatch = 4096;        // sequences per call (plan runs in one CTA)
constexpr int kMaxLen = 1 << 20;       // Lmax bound (TMA coordinates are int32)

__host__ __device__ constexpr int item_rows(int kind) { return kind == kKindFwd ? kFwdItemRows : kBwdItemRows; }

// Columns per block streamed by a backward kernel: 128, except 64 for dK/dV
// with d = 128 (its TMEM budget).
__host__ __device__ constexpr int bwd_col_block(bool kv, int d) { return (kv && d == 128) ? 64 : 128; }

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Valid length of sequence b, or 0 if the caller's value is outside [0, L]
// (the plan flags that case in the workspace header).
__device__ __forceinline__ int load_len(const int* lengths, int b, int L) {
  const int n = __ldg(lengths + b);
  return (n < 0 || n > L) ? 0 : n;
}

// One work item as the plan stores it: 16 bytes {b * H + h, row block, n_b,
// start_b}, so a kernel learns the item, its sequence's valid length and (for
// packed inputs) the sequence's first token from one load.
struct Item {
  int bh;     // b * H + h
  int blk;    // row-block index within the slice
  int n;      // valid length of sequence b
  int start;  // packed layout: index of the sequence's first token (0 when padded)
};

__device__ __forceinline__ Item load_item(const int* ws, int idx) {
  const int4 v = reinterpret_cast<const int4*>(ws + kHeaderWords)[idx];
  return Item{v.x, v.y, v.z, v.w};
}

// Where the rows of a (b, h) slice live, for both input layouts.
//  padded [B][H][Lmax][d]: TMA view {d, Lmax, B*H}; row r of slice bh is at
//    (y, z) = (r, bh). Rows n_b <= r < Lmax are padding and are written as zeros.
//  packed [total][H][d] (sequence b holds tokens start_b .. start_b + n_b - 1):
//    TMA view {d, H, total}; row r is at (y, z) = (h, start_b + r). Rows r >= n_b
//    belong to the next sequence and are never written.
template <bool PACKED>
struct RowMap {
  int H, L;
  __device__ __forceinline__ int y(const Item& it, int h, int row) const { return PACKED ? h : row; }
  __device__ __forceinline__ int z(const Item& it, int row) const { return PACKED ? it.start + row : it.bh; }
  // Element offset of the row in an output tensor of head size D.
  __device__ __forceinline__ size_t offset(const Item& it, int h, int row, int D) const {
    return PACKED ? (static_cast<size_t>(it.start + row) * H + h) * D : (static_cast<size_t>(it.bh) * L + row) * D;
  }
  // Whether the item's epilogue writes this row (zeros when row >= n).
  __device__ __forceinline__ bool writes(int row, int n) const { return PACKED ? row < n : row < L; }
};

constexpr Item kNoItem{0, 0, -1, 0};  // end of the work list

// Dynamic longest-processing-time-first scheduling. The plan lists the items
// longest first; each CTA's producer takes item blockIdx.x first and every
// later one from the claim counter in the workspace header, so a CTA gets the
// next item of the list when it is ready for one. The producer hands each
// item to the CTA's other roles through this two-slot ring in shared memory
// (so they never wait on a global load for it); after the last item it
// publishes kNoItem.
struct ItemRing {
  int4 slot[2];
  uint64_t full[2];   // count 1: the producer wrote the slot
  uint64_t empty[2];  // count = consumer arrivals per item
};

__device__ __forceinline__ void ring_init(ItemRing& r, int consumers) {
  for (int s = 0; s < 2; ++s) {
    mbar_init(&r.full[s], 1);
    mbar_init(&r.empty[s], consumers);
  }
}

// Producer: the CTA's next item (its first is `blockIdx.x`, `claimed` holds a
// counter value taken earlier, or -1 for the first call).
__device__ __forceinline__ Item next_item(const int* ws, int claimed, int count) {
  const int idx = claimed < 0 ? static_cast<int>(blockIdx.x) : claimed + static_cast<int>(gridDim.x);
  return idx < count ? load_item(ws, idx) : kNoItem;
}

__device__ __forceinline__ bool ring_publish(ItemRing& r, uint32_t& st, uint32_t& ph, const Item& item,
                                             volatile int* abort_flag, int* ws, int site) {
  if (!mbar_wait(&r.empty[st], ph ^ 1, abort_flag, ws, site)) return false;
  r.slot[st] = make_int4(item.bh, item.blk, item.n, item.start);
  mbar_arrive(&r.full[st]);
  if (++st == 2) { st = 0; ph ^= 1; }
  return true;
}

// Consumer side: wait for the next slot and copy the item out. A single
// consuming thread releases the slot with ring_release at once; a warp
// releases it once every lane has read it (__syncwarp, then lane 0).
__device__ __forceinline__ bool ring_read(ItemRing& r, uint32_t st, uint32_t ph, Item* item,
                                          volatile int* abort_flag, int* ws, int site) {
  if (!mbar_wait(&r.full[st], ph, abort_flag, ws, site)) return false;
  const int4 v = r.slot[st];  // ordered after the wait by its acquire and memory clobber
  *item = Item{v.x, v.y, v.z, v.w};
  return true;
}

__device__ __forceinline__ void ring_release(ItemRing& r, uint32_t& st, uint32_t& ph, bool arrive) {
  if (arrive) mbar_arrive(&r.empty[st]);
  if (++st == 2) { st = 0; ph ^= 1; }
}

// 1/sqrt(d) for the supported head sizes.
template <int D>
struct Scale;
template <>
struct Scale<64> {
  static constexpr float value = 0.125f;
};
template <>
struct Scale<128> {
  static constexpr float value = 0.08838834764831845f;
};

// sigma(s * scale + bias) for one score, written as 1/2 + tanh(x/2)/2 with the
// hardware tanh ("a hardware-optimised tanh approximation for the sigmoid",
// Better Models, Faster Training, sec. 2C). half_scale = scale/2 and
// half_bias = bias/2 are folded into one FMA.
__device__ __forceinline__ float sigmoid_from_score(float s, float half_scale, float half_bias) {
  const float t = tanh_approx(fmaf(s, half_scale, half_bias));
  return fmaf(t, 0.5f, 0.5f);
}

// Zero one unit of the output rows that no work item covers: rows
// [ceil(n_b/rows)*rows, L) of slice u / parts are cut into `parts` interleaved
// shares of 16-byte chunks, and this warp writes share u % parts of out0 (and
// out1).
__device__ __forceinline__ void zero_fill_unit(const int* lengths, int H, int L, int d, int rows, int parts,
                                               long long u, int lane, __nv_bfloat16* out0, __nv_bfloat16* out1) {
  const int slice = static_cast<int>(u / parts);
  const int part = static_cast<int>(u % parts);
  const int n = load_len(lengths, slice / H, L);
  const int cover = min(L, ceil_div(n, rows) * rows);
  const long long nchunks = static_cast<long long>(L - cover) * (d / 8);  // 16-byte chunks
  const size_t base = (static_cast<size_t>(slice) * L + cover) * d;
  uint4* p0 = reinterpret_cast<uint4*>(out0 + base);
  uint4* p1 = out1 ? reinterpret_cast<uint4*>(out1 + base) : nullptr;
  for (long long c = static_cast<long long>(part) * 32 + lane; c < nchunks; c += static_cast<long long>(parts) * 32) {
    p0[c] = make_uint4(0, 0, 0, 0);
    if (p1) p1[c] = make_uint4(0, 0, 0, 0);
  }
}

// The same rows cut into `parts` consecutive shares instead (the dQ kernel's
// fill, whose units go either to bulk copies or to warps): unit u covers the
// 16-byte chunks [begin, end) counted from element `base` of the output.
struct FillRange {
  size_t base;
  long long begin, end;
};

__device__ __forceinline__ FillRange zero_fill_range(const int* lengths, int H, int L, int d, int rows, int parts,
                                                     long long u) {
  const int slice = static_cast<int>(u / parts);
  const int part = static_cast<int>(u % parts);
  const int n = load_len(lengths, slice / H, L);
  const int cover = min(L, ceil_div(n, rows) * rows);
  const long long nchunks = static_cast<long long>(L - cover) * (d / 8);
  const long long share = (nchunks + parts - 1) / parts;
  FillRange f;
  f.base = (static_cast<size_t>(slice) * L + cover) * d;
  f.begin = min(nchunks, part * share);
  f.end = min(nchunks, f.begin + share);
  return f;
}

// One warp writes the zeros of a consecutive-share unit.
__device__ __forceinline__ void zero_fill_range_warp(const FillRange& f, int lane, __nv_bfloat16* out) {
  uint4* p = reinterpret_cast<uint4*>(out + f.base);
  for (long long c = f.begin + lane; c < f.end; c += 32) p[c] = make_uint4(0, 0, 0, 0);
}

// Shares per slice for the zero fill: enough units to spread over the SMs.
inline int zero_fill_parts(long long slices, int num_sms) {
  return static_cast<int>(std::max<long long>(1, std::min<long long>(64, (4LL * num_sms + slices - 1) / slices)));
}

// Store 64 bytes (one row's 32 bf16 values, packed in pairs) at dst, which is
// 16-byte aligned. An epilogue lane owns one row, so a warp's store touches 32
// rows; 32-byte stores halve the number of such instructions when dst is
// 32-byte aligned (warp-uniform: row strides are multiples of 32 bytes).
__device__ __forceinline__ void store_row64B(void* dst, const uint32_t (&w)[16]) {
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                       reinterpret_cast<uint8_t*>(dst) + 32 * h),
                   "r"(w[8 * h]), "r"(w[8 * h + 1]), "r"(w[8 * h + 2]), "r"(w[8 * h + 3]), "r"(w[8 * h + 4]),
                   "r"(w[8 * h + 5]), "r"(w[8 * h + 6]), "r"(w[8 * h + 7])
                   : "memory");
  } else {
    uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) p[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// sigma for long sequences. The bias -ln(n) puts the typical weight near 1/n;
// for n beyond kAccurateSigmoidLen the tanh route computes those weights just
// above tanh = -1, where the hardware tanh's absolute error becomes a relative
// error of several percent (measured: O rel-L2 1.1e-2 at n = 2^20). There
// sigma = 1 / (1 + 2^(-x log2 e)) is used instead: two MUFU operations (ex2,
// rcp) per score, relative error ~1e-6 everywhere. neg_scale_l2e = -scale *
// log2(e), neg_bias_l2e = ln(n) * log2(e) = log2(n).
constexpr int kAccurateSigmoidLen = 65536;

__device__ __forceinline__ float sigmoid_accurate(float s, float neg_scale_l2e, float neg_bias_l2e) {
  return rcp_approx(1.0f + ex2_approx(fmaf(s, neg_scale_l2e, neg_bias_l2e)));
}

// ACCURATE (a kernel template parameter, chosen per call from Lmax) selects
// sigmoid_accurate.
template <bool ACCURATE>
__device__ __forceinline__ float sigmoid_of(float s, float half_scale, float half_bias, float neg_scale_l2e,
                                            float neg_bias_l2e) {
  return ACCURATE ? sigmoid_accurate(s, neg_scale_l2e, neg_bias_l2e) : sigmoid_from_score(s, half_scale, half_bias);
}

// Convert 32 fp32 accumulator values (times `mul`) to bf16 and store them.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[32], float mul) {
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
  store_row64B(dst, w);
}

__device__ __forceinline__ void store_zero32(__nv_bfloat16* dst) {
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = 0u;
  store_row64B(dst, w);
}

// Launch `kernel` so that it may start while the previous kernel in `stream` is
// still running (programmatic stream serialization). The kernel calls
// grid_dep_wait() before it touches anything that earlier kernel writes.
template <typename... Params, typename... Args>
inline cudaError_t launch_programmatic(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                       cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace sigattn
