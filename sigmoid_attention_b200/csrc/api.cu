// api.cu -- the C ABI (include/sigattn.h): argument checks, TMA tensor maps and
// the launches of each call's kernels (plan; compute, with a programmatic
// dependency on the plan; for the padded layout the zero fill of uncovered
// output rows). No allocation, no host sync (except in sigattn_read_error,
// which exists to synchronise).
#include <climits>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/sigattn.h"
#include "common.cuh"

namespace sigattn {
cudaError_t launch_prep(const int* lengths, const int* cu, int total, int B, int H, int L, int kind, KeyRange kr,
                        int* ws, cudaStream_t stream);
cudaError_t launch_fill(const int* lengths, int B, int H, int L, int d, int kind, KeyRange kr, int elem_bytes,
                        void* out0, void* out1, int num_sms, cudaStream_t stream);
int plan_host(const int* lengths, int B, int H, int L, int kind, int* out, int cap);
cudaError_t launch_selftest_timeout(int* ws, unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_eval_sigmoid(const float* s, float* p, float* slope, int count, int d, int n, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_cast_bf16(const float* in, void* out, long long count, int num_sms, cudaStream_t stream);
cudaError_t launch_fwd(int d, bool packed, bool f32out, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, void* o, int* ws, int B, int H, int L, KeyRange kr, int num_sms,
                       cudaStream_t stream);
cudaError_t launch_softmax_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, int* ws,
                               int B, int H, int L, int num_sms, cudaStream_t stream);
cudaError_t launch_prep_bwd(const int* lengths, const int* cu, int total, int B, int H, int L, int* ws_dq,
                            int* ws_dkdv, cudaStream_t stream);
cudaError_t launch_bwd_dq(int d, bool packed, bool f32out, const CUtensorMap& tq, const CUtensorMap& tdo,
                          const CUtensorMap& tk, const CUtensorMap& tv, void* dq, int* ws, int B, int H, int L,
                          KeyRange kr, int num_sms, const int* fill_lengths, cudaStream_t stream,
                          const BwdLink& link = BwdLink{});
cudaError_t launch_bwd_dkdv(int d, bool packed, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                            const CUtensorMap& tdo, void* dk, void* dv, int* ws, int B, int H, int out_rows, int Lmax,
                            KeyRange kr, int num_sms, const int* fill_lengths, cudaStream_t stream,
                            const BwdLink& link = BwdLink{});
void set_last_error(const char* msg);
}  // namespace sigattn

using namespace sigattn;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

struct DeviceInfo {
  int num_sms = 0;
  bool supported = false;
};

// SM count and architecture check of the current device (cached per device).
bool device_info(DeviceInfo* out) {
  static DeviceInfo cache[64];
  static bool have[64] = {};
  static std::once_flag once[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  // A thread that has not used this library's CUDA runtime yet (for example
  // torch's autograd worker) may have no current context, which the tensor-map
  // encoder needs; cudaSetDevice makes the device's primary context current.
  thread_local int ready_for = -1;
  if (ready_for != dev) {
    if (cudaSetDevice(dev) != cudaSuccess) return false;
    ready_for = dev;
  }
  // Queried once per device (safely across host threads).
  std::call_once(once[dev], [dev] {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return;
    if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return;
    cache[dev].num_sms = sms;
    cache[dev].supported = (major == 10 && minor == 0);
    have[dev] = true;
  });
  if (!have[dev]) return false;
  *out = cache[dev];
  return true;
}

// 3-D view {d, Lmax, B*H} of a [B][H][Lmax][d] bf16 tensor, loaded as
// [box_rows rows][64 columns] boxes with the 128-byte swizzle the tcgen05
// descriptors expect. Rows past Lmax read as zeros.
bool make_map(CUtensorMap* map, const void* ptr, int BH, int L, int d, int box_rows = 128) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t elem[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view {d, H, total} of a packed [total][H][d] bf16 tensor, loaded as
// [box_rows tokens][1 head][64 columns] boxes (the same shared-memory image as
// a [box_rows][64] box). Tokens past `total` read as zeros.
bool make_map_packed(CUtensorMap* map, const void* ptr, int total, int H, int d, int box_rows = 128) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(total)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(H) * d * 2};
  const cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t elem[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, elem,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed token count bound: token coordinates start_b + row (row < n_b + 256)
// stay in int32.
constexpr int kMaxPackedTokens = INT_MAX - 4096;

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

long long max_items(int B, int H, int L) {
  return static_cast<long long>(B) * H * ceil_div(L, kBwdItemRows);
}

int check_sizes(int B, int H, int L, int d) {
  if (d != 64 && d != 128) return SIGATTN_ERR_UNSUPPORTED;
  if (B < 1 || H < 1 || L < 1) return SIGATTN_ERR_INVALID_ARG;
  if (B > kMaxBatch || L > kMaxLen) return SIGATTN_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > INT_MAX / 2 || max_items(B, H, L) > INT_MAX / 4)
    return SIGATTN_ERR_UNSUPPORTED;
  return SIGATTN_OK;
}

// Text of the last CUDA failure seen by this thread (see sigattn_last_error).
thread_local char g_last_error[160] = "no error";

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return SIGATTN_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
  return SIGATTN_ERR_CUDA;
}

}  // namespace

void sigattn::set_last_error(const char* msg) { snprintf(g_last_error, sizeof(g_last_error), "%s", msg); }

namespace {

int map_failure() {
  snprintf(g_last_error, sizeof(g_last_error), "cuTensorMapEncodeTiled failed or is unavailable");
  return SIGATTN_ERR_CUDA;
}

int check_call(int B, int H, int L, int d, const int32_t* lengths, const void* ws, size_t ws_bytes,
               DeviceInfo* info) {
  int st = check_sizes(B, H, L, d);
  if (st != SIGATTN_OK) return st;
  if (lengths == nullptr || (reinterpret_cast<uintptr_t>(lengths) & 3u) != 0) return SIGATTN_ERR_INVALID_ARG;
  if (!aligned16(ws) || ws_bytes < sigattn_workspace_size(B, H, L, d)) return SIGATTN_ERR_INVALID_ARG;
  if (!device_info(info)) {
    const cudaError_t e = cudaGetLastError();
    return cuda_status(e != cudaSuccess ? e : cudaErrorUnknown);
  }
  if (!info->supported) return SIGATTN_ERR_UNSUPPORTED;
  return SIGATTN_OK;
}

// The key range of a padded-layout call: 0 <= begin, 1 <= count and
// begin + count <= Lmax.
bool range_ok(KeyRange kr, int Lmax) {
  return kr.begin >= 0 && kr.count >= 1 && static_cast<long long>(kr.begin) + kr.count <= Lmax;
}

// Padded-layout forward over the keys kr (whole sequences: {0, Lmax}); k and
// v hold those keys only ([B][H][kr.count][d]); f32out writes o as fp32.
int fwd_padded(const void* q, const void* k, const void* v, void* o, bool f32out, const int32_t* lengths, int B,
               int H, int Lmax, int d, KeyRange kr, void* workspace, size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, Lmax, d, lengths, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (!range_ok(kr, Lmax)) return SIGATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SIGATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, B * H, Lmax, d) || !make_map(&tk, k, B * H, kr.count, d) ||
      !make_map(&tv, v, B * H, kr.count, d))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  st = cuda_status(launch_prep(lengths, nullptr, 0, B, H, Lmax, SIGATTN_KIND_FWD, kr, ws, s));
  if (st == SIGATTN_OK)
    st = cuda_status(launch_fwd(d, false, f32out, tq, tk, tv, o, ws, B, H, Lmax, kr, info.num_sms, s));
  if (st != SIGATTN_OK) return st;
  return cuda_status(
      launch_fill(lengths, B, H, Lmax, d, SIGATTN_KIND_FWD, kr, f32out ? 4 : 2, o, nullptr, info.num_sms, s));
}

int dq_padded(const void* q, const void* k, const void* v, const void* dout, void* dq, bool f32out,
              const int32_t* lengths, int B, int H, int Lmax, int d, KeyRange kr, void* workspace,
              size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, Lmax, d, lengths, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (!range_ok(kr, Lmax)) return SIGATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq))
    return SIGATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, q, B * H, Lmax, d) || !make_map(&tk, k, B * H, kr.count, d) ||
      !make_map(&tv, v, B * H, kr.count, d) || !make_map(&tdo, dout, B * H, Lmax, d))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  st = cuda_status(launch_prep(lengths, nullptr, 0, B, H, Lmax, SIGATTN_KIND_DQ, kr, ws, s));
  if (st != SIGATTN_OK) return st;
  // The dQ kernel zeroes dQ's uncovered padded rows itself.
  return cuda_status(
      launch_bwd_dq(d, false, f32out, tq, tdo, tk, tv, dq, ws, B, H, Lmax, kr, info.num_sms, lengths, s));
}

// dK, dV of the keys kr: k, v, dk, dv are [B][H][kr.count][d].
int dkdv_padded(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                const int32_t* lengths, int B, int H, int Lmax, int d, KeyRange kr, void* workspace,
                size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, Lmax, d, lengths, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (!range_ok(kr, Lmax)) return SIGATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return SIGATTN_ERR_INVALID_ARG;
  // K, V are the row operands (128-row boxes); Q, dO are streamed in blocks of
  // bwd_col_block(true, d) rows.
  const int cb = bwd_col_block(true, d);
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map(&tq, q, B * H, Lmax, d, cb) || !make_map(&tk, k, B * H, kr.count, d) ||
      !make_map(&tv, v, B * H, kr.count, d) || !make_map(&tdo, dout, B * H, Lmax, d, cb))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  st = cuda_status(launch_prep(lengths, nullptr, 0, B, H, Lmax, SIGATTN_KIND_DKDV, kr, ws, s));
  if (st != SIGATTN_OK) return st;
  // The dK/dV kernel zeroes the uncovered rows of dK and dV itself.
  return cuda_status(
      launch_bwd_dkdv(d, false, tk, tv, tq, tdo, dk, dv, ws, B, H, kr.count, Lmax, kr, info.num_sms, lengths, s));
}

// Bytes of one plan region (header and work list), rounded up to 256 so that
// the second region of a whole-backward workspace stays aligned.
size_t plan_region_bytes(int B, int H, int Lmax) {
  const size_t n = static_cast<size_t>(kHeaderWords) * 4 + static_cast<size_t>(max_items(B, H, Lmax)) * 16;
  return (n + 255) / 256 * 256;
}

// dQ, dK and dV in one call: one plan launch builds both work lists (dQ's in
// the workspace's first region, dK/dV's in the second), then the dQ kernel
// and the dK/dV kernel, which takes SMs as the dQ kernel's CTAs finish and
// completes after it (bwd.cu). Errors of both go to the first header.
// Padded layout: lengths, L = Lmax; packed: cu_seqlens, L = max_seqlen and
// `total` tokens.
int bwd_whole(bool packed, const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk,
              void* dv, const int32_t* lengths_or_cu, int B, int H, int L, int total, int d, void* workspace,
              size_t workspace_bytes, void* stream) {
  if (workspace_bytes < sigattn_bwd_workspace_size(B, H, L, d)) return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  int st = check_call(B, H, L, d, lengths_or_cu, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (packed && (total < 1 || total > kMaxPackedTokens))
    return total < 1 ? SIGATTN_ERR_INVALID_ARG : SIGATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return SIGATTN_ERR_INVALID_ARG;
  const int cb = bwd_col_block(true, d);
  auto map = [&](CUtensorMap* m, const void* p, int box_rows) {
    return packed ? make_map_packed(m, p, total, H, d, box_rows) : make_map(m, p, B * H, L, d, box_rows);
  };
  CUtensorMap tq, tk, tv, tdo, tq_c, tdo_c;
  if (!map(&tq, q, 128) || !map(&tk, k, 128) || !map(&tv, v, 128) || !map(&tdo, dout, 128) || !map(&tq_c, q, cb) ||
      !map(&tdo_c, dout, cb))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws_dq = static_cast<int*>(workspace);
  int* ws_dkdv = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + plan_region_bytes(B, H, L));
  const KeyRange all{0, L};
  const int32_t* lengths = packed ? nullptr : lengths_or_cu;
  st = cuda_status(launch_prep_bwd(lengths, packed ? lengths_or_cu : nullptr, packed ? total : 0, B, H, L, ws_dq,
                                   ws_dkdv, s));
  if (st == SIGATTN_OK)
    st = cuda_status(launch_bwd_dq(d, packed, false, tq, tdo, tk, tv, dq, ws_dq, B, H, L, all, info.num_sms,
                                   lengths, s));
  if (st != SIGATTN_OK) return st;
  BwdLink link;
  link.err = ws_dq;
  link.overlap = true;
  return cuda_status(launch_bwd_dkdv(d, packed, tk, tv, tq_c, tdo_c, dk, dv, ws_dkdv, B, H, L, L, all,
                                     info.num_sms, lengths, s, link));
}

}  // namespace

namespace sigattn {

// The host checks of a padded-layout forward call that do not involve a
// workspace: sizes, the lengths pointer, 16-byte alignment of q, k, v, o and
// the device's architecture (for entry points that bring their own scratch).
int check_fwd_inputs(const void* q, const void* k, const void* v, const void* o, const int32_t* lengths, int B,
                     int H, int L, int d) {
  int st = check_sizes(B, H, L, d);
  if (st != SIGATTN_OK) return st;
  if (lengths == nullptr || (reinterpret_cast<uintptr_t>(lengths) & 3u) != 0) return SIGATTN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) {
    const cudaError_t e = cudaGetLastError();
    return cuda_status(e != cudaSuccess ? e : cudaErrorUnknown);
  }
  return info.supported ? SIGATTN_OK : SIGATTN_ERR_UNSUPPORTED;
}

// SIGATTN_OK for cudaSuccess; otherwise records the error's text for
// sigattn_last_error and returns SIGATTN_ERR_CUDA.
int report_cuda(cudaError_t e) { return cuda_status(e); }

}  // namespace sigattn

extern "C" {

int sigattn_version(void) { return 100; }

const char* sigattn_status_str(int status) {
  switch (status) {
    case SIGATTN_OK: return "ok";
    case SIGATTN_ERR_INVALID_ARG: return "invalid argument";
    case SIGATTN_ERR_UNSUPPORTED: return "unsupported size or device";
    case SIGATTN_ERR_CUDA: return "CUDA error";
    case SIGATTN_ERR_TIMEOUT: return "kernel wait timed out";
    default: return "unknown status";
  }
}

int sigattn_block_rows(int kind) {
  if (kind < SIGATTN_KIND_FWD || kind > SIGATTN_KIND_DKDV) return -1;
  return item_rows(kind);
}

size_t sigattn_workspace_size(int B, int H, int Lmax, int d) {
  if (check_sizes(B, H, Lmax, d) != SIGATTN_OK) return 0;
  return static_cast<size_t>(kHeaderWords) * 4 + static_cast<size_t>(max_items(B, H, Lmax)) * 16;
}

size_t sigattn_bwd_workspace_size(int B, int H, int Lmax, int d) {
  if (check_sizes(B, H, Lmax, d) != SIGATTN_OK) return 0;
  return 2 * plan_region_bytes(B, H, Lmax);
}

int sigattn_bwd(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk, void* dv,
                const int32_t* lengths, int B, int H, int Lmax, int d, void* workspace, size_t workspace_bytes,
                void* stream) {
  return bwd_whole(false, q, k, v, dout, dq, dk, dv, lengths, B, H, Lmax, 0, d, workspace, workspace_bytes, stream);
}

int sigattn_bwd_varlen(const void* q, const void* k, const void* v, const void* dout, void* dq, void* dk, void* dv,
                       const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total, int d, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return bwd_whole(true, q, k, v, dout, dq, dk, dv, cu_seqlens, B, H, max_seqlen, total, d, workspace,
                   workspace_bytes, stream);
}

int sigattn_fwd(const void* q, const void* k, const void* v, void* o, const int32_t* lengths, int B, int H,
                int Lmax, int d, void* workspace, size_t workspace_bytes, void* stream) {
  return fwd_padded(q, k, v, o, false, lengths, B, H, Lmax, d, KeyRange{0, Lmax}, workspace, workspace_bytes, stream);
}

int sigattn_fwd_partial(const void* q, const void* k, const void* v, float* o_partial, const int32_t* lengths, int B,
                        int H, int Lmax, int d, int key_begin, int key_count, void* workspace, size_t workspace_bytes,
                        void* stream) {
  return fwd_padded(q, k, v, o_partial, true, lengths, B, H, Lmax, d, KeyRange{key_begin, key_count}, workspace,
                    workspace_bytes, stream);
}

int sigattn_bwd_dq(const void* q, const void* k, const void* v, const void* dout, void* dq, const int32_t* lengths,
                   int B, int H, int Lmax, int d, void* workspace, size_t workspace_bytes, void* stream) {
  return dq_padded(q, k, v, dout, dq, false, lengths, B, H, Lmax, d, KeyRange{0, Lmax}, workspace, workspace_bytes,
                   stream);
}

int sigattn_bwd_dq_partial(const void* q, const void* k, const void* v, const void* dout, float* dq_partial,
                           const int32_t* lengths, int B, int H, int Lmax, int d, int key_begin, int key_count,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return dq_padded(q, k, v, dout, dq_partial, true, lengths, B, H, Lmax, d, KeyRange{key_begin, key_count}, workspace,
                   workspace_bytes, stream);
}

int sigattn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                     const int32_t* lengths, int B, int H, int Lmax, int d, void* workspace, size_t workspace_bytes,
                     void* stream) {
  return dkdv_padded(q, k, v, dout, dk, dv, lengths, B, H, Lmax, d, KeyRange{0, Lmax}, workspace, workspace_bytes,
                     stream);
}

int sigattn_bwd_dkdv_range(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                           const int32_t* lengths, int B, int H, int Lmax, int d, int key_begin, int key_count,
                           void* workspace, size_t workspace_bytes, void* stream) {
  return dkdv_padded(q, k, v, dout, dk, dv, lengths, B, H, Lmax, d, KeyRange{key_begin, key_count}, workspace,
                     workspace_bytes, stream);
}

int sigattn_softmax_fwd(const void* q, const void* k, const void* v, void* o, const int32_t* lengths, int B, int H,
                        int Lmax, int d, void* workspace, size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, Lmax, d, lengths, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (d != 64) return SIGATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SIGATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, B * H, Lmax, d) || !make_map(&tk, k, B * H, Lmax, d) || !make_map(&tv, v, B * H, Lmax, d))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  const KeyRange all{0, Lmax};
  st = cuda_status(launch_prep(lengths, nullptr, 0, B, H, Lmax, SIGATTN_KIND_FWD, all, ws, s));
  if (st == SIGATTN_OK) st = cuda_status(launch_softmax_fwd(tq, tk, tv, o, ws, B, H, Lmax, info.num_sms, s));
  if (st != SIGATTN_OK) return st;
  return cuda_status(launch_fill(lengths, B, H, Lmax, d, SIGATTN_KIND_FWD, all, 2, o, nullptr, info.num_sms, s));
}

int sigattn_cast_bf16(const float* x, void* y, long long count, void* stream) {
  if (count < 0 || count % 8 != 0) return SIGATTN_ERR_INVALID_ARG;
  if (count == 0) return SIGATTN_OK;
  if (!aligned16(x) || !aligned16(y)) return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return cuda_status(cudaErrorUnknown);
  if (!info.supported) return SIGATTN_ERR_UNSUPPORTED;
  return cuda_status(launch_cast_bf16(x, y, count, info.num_sms, static_cast<cudaStream_t>(stream)));
}

int sigattn_fwd_varlen(const void* q, const void* k, const void* v, void* o, const int32_t* cu_seqlens, int B,
                       int H, int max_seqlen, int total, int d, void* workspace, size_t workspace_bytes,
                       void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, max_seqlen, d, cu_seqlens, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (total < 1 || total > kMaxPackedTokens) return total < 1 ? SIGATTN_ERR_INVALID_ARG : SIGATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SIGATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv;
  if (!make_map_packed(&tq, q, total, H, d) || !make_map_packed(&tk, k, total, H, d) ||
      !make_map_packed(&tv, v, total, H, d))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  const KeyRange all{0, max_seqlen};
  st = cuda_status(launch_prep(nullptr, cu_seqlens, total, B, H, max_seqlen, SIGATTN_KIND_FWD, all, ws, s));
  if (st != SIGATTN_OK) return st;
  return cuda_status(launch_fwd(d, true, false, tq, tk, tv, o, ws, B, H, max_seqlen, all, info.num_sms, s));
}

int sigattn_bwd_dq_varlen(const void* q, const void* k, const void* v, const void* dout, void* dq,
                          const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total, int d, void* workspace,
                          size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, max_seqlen, d, cu_seqlens, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (total < 1 || total > kMaxPackedTokens) return total < 1 ? SIGATTN_ERR_INVALID_ARG : SIGATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq))
    return SIGATTN_ERR_INVALID_ARG;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_packed(&tq, q, total, H, d) || !make_map_packed(&tk, k, total, H, d) ||
      !make_map_packed(&tv, v, total, H, d) || !make_map_packed(&tdo, dout, total, H, d))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  const KeyRange all{0, max_seqlen};
  st = cuda_status(launch_prep(nullptr, cu_seqlens, total, B, H, max_seqlen, SIGATTN_KIND_DQ, all, ws, s));
  if (st != SIGATTN_OK) return st;
  return cuda_status(
      launch_bwd_dq(d, true, false, tq, tdo, tk, tv, dq, ws, B, H, max_seqlen, all, info.num_sms, nullptr, s));
}

int sigattn_bwd_dkdv_varlen(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                            const int32_t* cu_seqlens, int B, int H, int max_seqlen, int total, int d,
                            void* workspace, size_t workspace_bytes, void* stream) {
  DeviceInfo info;
  int st = check_call(B, H, max_seqlen, d, cu_seqlens, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  if (total < 1 || total > kMaxPackedTokens) return total < 1 ? SIGATTN_ERR_INVALID_ARG : SIGATTN_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dk) || !aligned16(dv))
    return SIGATTN_ERR_INVALID_ARG;
  const int cb = bwd_col_block(true, d);
  CUtensorMap tq, tk, tv, tdo;
  if (!make_map_packed(&tq, q, total, H, d, cb) || !make_map_packed(&tk, k, total, H, d) ||
      !make_map_packed(&tv, v, total, H, d) || !make_map_packed(&tdo, dout, total, H, d, cb))
    return map_failure();
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* ws = static_cast<int*>(workspace);
  const KeyRange all{0, max_seqlen};
  st = cuda_status(launch_prep(nullptr, cu_seqlens, total, B, H, max_seqlen, SIGATTN_KIND_DKDV, all, ws, s));
  if (st != SIGATTN_OK) return st;
  return cuda_status(launch_bwd_dkdv(d, true, tk, tv, tq, tdo, dk, dv, ws, B, H, max_seqlen, max_seqlen, all,
                                     info.num_sms, nullptr, s));
}

int sigattn_plan(const int32_t* lengths, int B, int H, int Lmax, int d, int kind, void* workspace,
                 size_t workspace_bytes, void* stream) {
  if (kind < SIGATTN_KIND_FWD || kind > SIGATTN_KIND_DKDV) return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  int st = check_call(B, H, Lmax, d, lengths, workspace, workspace_bytes, &info);
  if (st != SIGATTN_OK) return st;
  return cuda_status(launch_prep(lengths, nullptr, 0, B, H, Lmax, kind, KeyRange{0, Lmax}, static_cast<int*>(workspace),
                                 static_cast<cudaStream_t>(stream)));
}

int sigattn_plan_host(const int32_t* lengths_host, int B, int H, int Lmax, int kind, int32_t* items_out, int cap,
                      int* count) {
  if (kind < SIGATTN_KIND_FWD || kind > SIGATTN_KIND_DKDV) return SIGATTN_ERR_INVALID_ARG;
  if (lengths_host == nullptr || count == nullptr || cap < 0 || (cap > 0 && items_out == nullptr))
    return SIGATTN_ERR_INVALID_ARG;
  const int st = check_sizes(B, H, Lmax, 64);
  if (st != SIGATTN_OK) return st;
  *count = plan_host(lengths_host, B, H, Lmax, kind, items_out, cap);
  return SIGATTN_OK;
}

const char* sigattn_last_error(void) { return g_last_error; }

int sigattn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, int limit_us, void* stream) {
  if (!aligned16(workspace) || workspace_bytes < static_cast<size_t>(kHeaderWords) * 4 || limit_us < 1 ||
      limit_us > 10000000)
    return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return cuda_status(cudaErrorUnknown);
  if (!info.supported) return SIGATTN_ERR_UNSUPPORTED;
  return cuda_status(launch_selftest_timeout(static_cast<int*>(workspace),
                                             static_cast<unsigned long long>(limit_us) * 1000ull,
                                             static_cast<cudaStream_t>(stream)));
}

int sigattn_eval_sigmoid(const float* scores, float* p, float* slope, int count, int d, int n, void* stream) {
  if (d != 64 && d != 128) return SIGATTN_ERR_UNSUPPORTED;
  if (count < 0 || n < 1 || n > kMaxLen) return SIGATTN_ERR_INVALID_ARG;
  if (count == 0) return SIGATTN_OK;
  const auto aligned4 = [](const void* ptr) { return ptr != nullptr && (reinterpret_cast<uintptr_t>(ptr) & 3u) == 0; };
  if (!aligned4(scores) || !aligned4(p) || !aligned4(slope)) return SIGATTN_ERR_INVALID_ARG;
  DeviceInfo info;
  if (!device_info(&info)) return cuda_status(cudaErrorUnknown);
  if (!info.supported) return SIGATTN_ERR_UNSUPPORTED;
  return cuda_status(launch_eval_sigmoid(scores, p, slope, count, d, n, info.num_sms, static_cast<cudaStream_t>(stream)));
}

int sigattn_read_error(void* workspace, int* site, void* stream) {
  if (!aligned16(workspace)) return SIGATTN_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int hdr[2] = {0, 0};
  cudaError_t e = cudaMemcpyAsync(hdr, workspace, sizeof(hdr), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(workspace, 0, sizeof(hdr), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_status(e);
  if (site) *site = hdr[kHdrErrorSite];
  return hdr[kHdrError];
}

}  // extern "C"
