// C ABI of the exact-attention library: argument validation, TMA tensor maps, launches
// and the device status word.  The kernels are included here so that the whole library
// is one translation unit (the status word needs no relocatable device code).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"

#include "fwd_kernel.cuh"
#include "fwd256_kernel.cuh"
#include "fp8_ops.cuh"
#include "fwd_fp8_kernel.cuh"
#include "bwd_kernel.cuh"
#include "bwd256_kernel.cuh"
#include "decode_ops.cuh"
#include "decode_kernel.cuh"

namespace fa {
namespace {

constexpr unsigned long long kDefaultWaitLimitNs = 4000000000ull;
unsigned long long g_wait_limit_ns = kDefaultWaitLimitNs;

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// A bf16 [B, heads, rows, d] array with element strides st (d contiguous) viewed as the 4-D
// tensor (d, rows, heads, B); box = 64 columns x box_rows rows of one head, 128-byte swizzled.
// Rows past the end of a head read as zero.
bool make_map_bf16(CUtensorMap* map, const void* base, int d, int rows, int heads, int B, Strides st,
                   int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(heads), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(st.n) * 2, cuuint64_t(st.h) * 2, cuuint64_t(st.b) * 2};
  cuuint32_t box[4] = {64, cuuint32_t(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A one-byte (E4M3 code) packed array [B, heads, rows, x] as the 4-D tensor (x, rows, heads, B),
// box = 128 x 128, 128-byte swizzled; outside the tensor reads as zero.
bool make_map_u8(CUtensorMap* map, const void* base, int x, int rows, int heads, int B) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {cuuint64_t(x), cuuint64_t(rows), cuuint64_t(heads), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(x), cuuint64_t(x) * rows, cuuint64_t(x) * rows * heads};
  cuuint32_t box[4] = {128, 128, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The decode kernel's E4M3 K or V cache [B, heads, rows, d] with element strides st as the 4-D
// tensor (d, rows, heads, B): boxes of 16 rows x 128 codes, 128-byte swizzled, or at d = 64 of
// 16 unswizzled 64-byte rows.  Rows past the end read as zero.
bool make_map_dec_u8(CUtensorMap* map, const void* base, int d, int rows, int heads, int B, Strides st) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(rows), cuuint64_t(heads), cuuint64_t(B)};
  cuuint64_t strides[3] = {cuuint64_t(st.n), cuuint64_t(st.h), cuuint64_t(st.b)};
  cuuint32_t box[4] = {cuuint32_t(d >= 128 ? 128 : 64), cuuint32_t(kDecKeys), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, d >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The backward's fp32 dQ accumulator [BH, Np, d] as the 4-D tensor (d, Np, BH, 1) that its
// tensor reductions add into: 32 x 32 boxes (128-byte rows), 128-byte swizzled.
bool make_map_dq_acc(CUtensorMap* map, float* base, int d, long long Np, long long BH) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {cuuint64_t(d), cuuint64_t(Np), cuuint64_t(BH), 1};
  cuuint64_t strides[3] = {cuuint64_t(d) * 4, cuuint64_t(Np) * d * 4, cuuint64_t(BH) * Np * d * 4};
  cuuint32_t box[4] = {32, 32, 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// strides of a contiguous [B, heads, N, d] array
Strides packed(int heads, int N, int d) {
  return Strides{(long long)heads * N * d, (long long)N * d, (long long)d};
}

// every stride a positive multiple of 8 elements (16 bytes: TMA and the vector stores)
bool strides_ok(const Strides& s) {
  return s.b > 0 && s.h > 0 && s.n > 0 && s.b % 8 == 0 && s.h % 8 == 0 && s.n % 8 == 0;
}

// ---------------------------------------------------------------- validation
constexpr int kMaxDevices = 64;

int check_device() {
  static int ok_cache[kMaxDevices] = {0};  // 0 unknown, 1 ok, 2 wrong device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return FA_ERR_DEVICE;
  if (ok_cache[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return FA_ERR_CUDA;
    ok_cache[dev] = (major == 10 && minor == 0) ? 1 : 2;
  }
  return ok_cache[dev] == 1 ? FA_OK : FA_ERR_DEVICE;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// A kernel that moves registers between its warpgroups (setmaxnreg) must be launched with at
// least `regs` registers per thread: the raised budgets come out of the launch share, and a raise
// the CTA cannot cover would wait forever.  Checked once per kernel and device.
// (The kernel is a template argument, so that each kernel has its own cache: instantiations
// share a function-pointer type.)
template <auto Kernel>
int check_launch_regs(int regs) {
  static int cache[kMaxDevices] = {0};   // 0 unknown, 1 ok, 2 too few
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FA_ERR_CUDA;
  if (cache[dev] == 0) {
    cudaFuncAttributes a;
    if (cudaFuncGetAttributes(&a, Kernel) != cudaSuccess) return FA_ERR_CUDA;
    cache[dev] = a.numRegs >= regs ? 1 : 2;
  }
  return cache[dev] == 1 ? FA_OK : FA_ERR_INTERNAL;
}

int check_problem(int B, int H, int N, int d, float scale, int causal, int window) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_SHAPE;
  const long long bh = (long long)B * H;
  const long long tiles = (N + kBlockM - 1) / kBlockM;
  if (bh > 0x7fffffffLL || bh * tiles > 0x7fffffffLL) return FA_ERR_SHAPE;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_HEADDIM;
  if (!(causal == 0 || causal == 1) || window < 0) return FA_ERR_MASK;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_SCALE;
  return FA_OK;
}

// query heads H read K/V heads H_kv in contiguous groups
int check_kv_heads(int H, int H_kv) { return (H_kv >= 1 && H_kv <= H && H % H_kv == 0) ? FA_OK : FA_ERR_SHAPE; }

template <class Kernel>
int set_smem(Kernel k, int bytes) {
  return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess ? FA_OK
                                                                                                     : FA_ERR_CUDA;
}

// launch a kernel that moves registers between its warpgroups, once its launch share is checked
template <auto Kernel, class... Args>
int launch_regs_checked(unsigned grid, unsigned threads, int smem, cudaStream_t stream, int regs,
                        const Args&... args) {
  if (set_smem(Kernel, smem) != FA_OK) return FA_ERR_CUDA;
  if (int rs = check_launch_regs<Kernel>(regs); rs != FA_OK) return rs;
  Kernel<<<grid, threads, smem, stream>>>(args...);
  return FA_OK;
}

// tensor maps and parameters of the d = 64 / 128 forward (fwd_kernel.cuh)
template <int D>
bool fwd_setup(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
               const Strides* st, float scale, int causal, int window, CUtensorMap* tq, CUtensorMap* tk,
               CUtensorMap* tv, FwdParams* prm) {
  if (!make_map_bf16(tq, q, D, N, H, B, st[0], kBlockM) || !make_map_bf16(tk, k, D, N, H_kv, B, st[1], kBlockN) ||
      !make_map_bf16(tv, v, D, N, H_kv, B, st[2], kBlockN))
    return false;
  prm->o = static_cast<__nv_bfloat16*>(o);
  prm->lse = lse;
  prm->N = N;
  prm->BH = B * H;
  prm->H = H;
  prm->group = H / H_kv;
  prm->o_st = st[3];
  prm->n_pairs = ((N + kBlockM - 1) / kBlockM + kQTiles - 1) / kQTiles;
  prm->causal = causal;
  prm->window = window > N ? N : window;   // a band of N or more keys is no band at all
  prm->scale_log2 = scale * 1.4426950408889634f;
  prm->wait_limit_ns = g_wait_limit_ns;
  return true;
}

// at least 120 KB of shared memory so that one CTA (and its 512 TMEM columns) owns the SM
constexpr int fwd_smem_bytes(int struct_bytes) {
  return struct_bytes + 1024 > 120 * 1024 ? struct_bytes + 1024 : 120 * 1024;
}

template <int D>
int launch_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
               const Strides* st, float scale, int causal, int window, cudaStream_t stream) {
  CUtensorMap tq, tk, tv, to;
  FwdParams prm;
  if (!fwd_setup<D>(q, k, v, o, lse, B, H, H_kv, N, st, scale, causal, window, &tq, &tk, &tv, &prm) ||
      !make_map_bf16(&to, o, D, N, H, B, st[3], kBlockM))
    return FA_ERR_CUDA;
  const int smem = fwd_smem_bytes(int(sizeof(FwdSmem<D>)));
  if (set_smem(fa_fwd_kernel<D>, smem) != FA_OK) return FA_ERR_CUDA;
  const unsigned grid = unsigned(prm.n_pairs) * unsigned(prm.BH);
  fa_fwd_kernel<D><<<grid, kFwdThreads, smem, stream>>>(tq, tk, tv, to, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// head dimension 256: one 128-row query tile per CTA, 64-key K/V tiles (fwd256_kernel.cuh)
int launch_fwd256(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
                  const Strides* st, float scale, int causal, int window, cudaStream_t stream) {
  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (!make_map_bf16(&tq, q, kD256, N, H, B, st[0], k256BlockM) ||
      !make_map_bf16(&tk, k, kD256, N, H_kv, B, st[1], k256BlockN) ||
      !make_map_bf16(&tv, v, kD256, N, H_kv, B, st[2], k256BlockN))
    return FA_ERR_CUDA;
  FwdParams prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.N = N;
  prm.BH = BH;
  prm.H = H;
  prm.group = H / H_kv;
  prm.o_st = st[3];
  prm.n_pairs = (N + k256BlockM - 1) / k256BlockM;   // query tiles per head
  prm.causal = causal;
  prm.window = window > N ? N : window;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = g_wait_limit_ns;
  static_assert(sizeof(Fwd256Smem) + 1024 <= 232448, "d = 256 forward shared memory exceeds 227 KB");
  const int smem = int(sizeof(Fwd256Smem)) + 1024;
  if (set_smem(fa_fwd256_kernel, smem) != FA_OK) return FA_ERR_CUDA;
  fa_fwd256_kernel<<<unsigned(prm.n_pairs) * unsigned(BH), k256Threads, smem, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// FP8 forward: q8, k8 [B, heads, N, 128] and vt8 [B, H_kv, 128, N] E4M3 codes, packed
int launch_fwd_fp8(const void* q8, const void* k8, const void* vt8, float q_scale, float k_scale, float v_scale,
                   void* o, float* lse, int B, int H, int H_kv, int N, float scale, int causal, int window,
                   cudaStream_t stream) {
  CUtensorMap tq, tk, tvt;
  if (!make_map_u8(&tq, q8, kF8D, N, H, B) || !make_map_u8(&tk, k8, kF8D, N, H_kv, B) ||
      !make_map_u8(&tvt, vt8, N, kF8D, H_kv, B))
    return FA_ERR_CUDA;
  FwdParams prm;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.N = N;
  prm.BH = B * H;
  prm.H = H;
  prm.group = H / H_kv;
  prm.o_st = packed(H, N, kF8D);
  prm.n_pairs = ((N + kBlockM - 1) / kBlockM + kQTiles - 1) / kQTiles;
  prm.causal = causal;
  prm.window = window > N ? N : window;
  prm.scale_log2 = scale * q_scale * k_scale * 1.4426950408889634f;
  prm.wait_limit_ns = g_wait_limit_ns;
  const int smem = int(sizeof(FwdFp8Smem)) + 1024;
  if (set_smem(fa_fwd_fp8_kernel, smem) != FA_OK) return FA_ERR_CUDA;
  fa_fwd_fp8_kernel<<<unsigned(prm.n_pairs) * unsigned(prm.BH), kFwdThreads, smem, stream>>>(tq, tk, tvt, prm, v_scale);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ---------------------------------------------------------------- backward
constexpr int kBwdPhasePrep = 1, kBwdPhaseMain = 2, kBwdPhaseFinal = 4, kBwdAllPhases = 7;

long long padded_rows(int N) { return ((long long)N + kBwdRows - 1) / kBwdRows * kBwdRows; }

size_t bwd_workspace_bytes(long long BH, int N, int d) {
  return size_t(4) * size_t(BH) * size_t(padded_rows(N)) * size_t(2 + d);
}

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
               void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, const Strides* st, float scale,
               int causal, int window, void* ws, cudaStream_t stream, int phases = kBwdAllPhases) {
  // st: q, k, v, o, dO, dq, dk, dv
  const int BH = B * H, BH_kv = B * H_kv;
  const long long Np = padded_rows(N);
  float* lp = static_cast<float*>(ws);
  float* dd = lp + size_t(BH) * Np;
  float* dq_acc = dd + size_t(BH) * Np;
  constexpr int G = D / 8;
  if (phases & kBwdPhasePrep) {
    const long long rows = (long long)BH * Np;
    const long long blocks = (rows + (256 / G) - 1) / (256 / G);
    fa_bwd_prep<D><<<unsigned(blocks), 256, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(dout), lse, lp, dd, dq_acc, N,
        int(Np), H, st[3], st[4], rows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (phases & kBwdPhaseMain) {
  CUtensorMap tq, tk, tv, tdo;
  constexpr int box_keys = D == 256 ? kB256Keys : kBwdKeys;
  if (!make_map_bf16(&tq, q, D, N, H, B, st[0], kBwdRows) || !make_map_bf16(&tk, k, D, N, H_kv, B, st[1], box_keys) ||
      !make_map_bf16(&tv, v, D, N, H_kv, B, st[2], box_keys) || !make_map_bf16(&tdo, dout, D, N, H, B, st[4], kBwdRows))
    return FA_ERR_CUDA;
  BwdParams prm;
  prm.lp = lp;
  prm.dd = dd;
  prm.dq_acc = dq_acc;
  prm.dk = static_cast<__nv_bfloat16*>(dk);
  prm.dv = static_cast<__nv_bfloat16*>(dv);
  prm.N = N;
  prm.Np = int(Np);
  prm.BH = BH;
  prm.H = H;
  prm.H_kv = H_kv;
  prm.group = H / H_kv;
  prm.dk_st = st[6];
  prm.dv_st = st[7];
  prm.n_kv_tiles = (N + kBwdKeys - 1) / kBwdKeys;
  prm.causal = causal;
  prm.window = window > N ? N : window;   // a band of N or more keys is no band at all
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.scale = scale;
  prm.wait_limit_ns = g_wait_limit_ns;
  if constexpr (D == 256) {
    // one CTA per (K/V head, 64-key tile): bwd256_kernel.cuh
    prm.n_kv_tiles = (N + kB256Keys - 1) / kB256Keys;
    static_assert(sizeof(Bwd256Smem) <= 232448, "d = 256 backward shared memory exceeds 227 KB");
    const int smem = int(sizeof(Bwd256Smem));
    CUtensorMap tdq;
    if (!make_map_dq_acc(&tdq, dq_acc, D, Np, BH)) return FA_ERR_CUDA;
    if (set_smem(fa_bwd256_kernel, smem) != FA_OK) return FA_ERR_CUDA;
    fa_bwd256_kernel<<<unsigned(prm.n_kv_tiles) * unsigned(BH_kv), kB256Threads, smem, stream>>>(tq, tk, tv, tdo,
                                                                                                         tdq, prm);
  } else {
    static_assert(sizeof(BwdSmem<D>) <= 232448, "backward shared memory exceeds 227 KB");
    const int smem = int(sizeof(BwdSmem<D>));   // the kernel checks that the base is 1 KB aligned
    CUtensorMap tdq, tdk, tdv;
    if (!make_map_dq_acc(&tdq, dq_acc, D, Np, BH) || !make_map_bf16(&tdk, dk, D, N, H_kv, B, st[6], 32) ||
        !make_map_bf16(&tdv, dv, D, N, H_kv, B, st[7], 32))
      return FA_ERR_CUDA;
    // one CTA per (K/V head, key tile); dK from the shared-memory dS when K/V heads are shared
    const unsigned grid = unsigned(prm.n_kv_tiles) * unsigned(BH_kv);
    const int rs = prm.group > 1 ? launch_regs_checked<fa_bwd_kernel<D, true>>(grid, kBwdThreads, smem, stream,
                                                                               kBwdLaunchRegs, tq, tk, tv, tdo, tdq,
                                                                               tdk, tdv, prm)
                                 : launch_regs_checked<fa_bwd_kernel<D, false>>(grid, kBwdThreads, smem, stream,
                                                                                kBwdLaunchRegs, tq, tk, tv, tdo, tdq,
                                                                                tdk, tdv, prm);
    if (rs != FA_OK) return rs;
  }
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  if (phases & kBwdPhaseFinal) {
    const long long rows = (long long)BH * N;
    const long long blocks = (rows + (256 / G) - 1) / (256 / G);
    fa_bwd_dq_final<D><<<unsigned(blocks), 256, 0, stream>>>(dq_acc, static_cast<__nv_bfloat16*>(dq), N, int(Np),
                                                             scale, H, st[5], rows);
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// ---------------------------------------------------------------- decode (few rows, many keys)
// Validates a decode problem and returns its plan (window clamped to N_k first).
int check_decode(int B, int H, int H_kv, int Nq, int Nk, int d, float scale, int causal, int window, DecPlan* pl) {
  if (B < 1 || H < 1 || H_kv < 1 || Nq < 1 || Nk < 1 || Nq > Nk) return FA_ERR_SHAPE;
  if (check_kv_heads(H, H_kv) != FA_OK) return FA_ERR_SHAPE;
  if (d != 64 && d != 128 && d != 256) return FA_ERR_HEADDIM;
  if (!(causal == 0 || causal == 1) || window < 0) return FA_ERR_MASK;
  if (!std::isfinite(scale) || !(scale > 0.f)) return FA_ERR_SCALE;
  const long long rows = (long long)(H / H_kv) * Nq;
  if (rows > 0x7fffffffLL - kDecRows || (long long)B * H * Nq > 0x7fffffffLL) return FA_ERR_SHAPE;
  *pl = dec_plan(B, H, H_kv, Nq, Nk, d, causal, window > Nk ? Nk : window);
  if (pl->ctas > 0x7fffffffLL) return FA_ERR_SHAPE;
  return FA_OK;
}

// k, v: bf16 arrays, or (kFp8) E4M3 codes with K = k_scale K8, V = v_scale V8.
template <int D, bool kFp8>
int launch_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int Nq,
                  int Nk, const Strides* st, float scale, int causal, int window, void* ws, const DecPlan& pl,
                  cudaStream_t stream, float k_scale = 1.f, float v_scale = 1.f) {
  DecParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.v_scale = v_scale;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.o_part = static_cast<float*>(ws);
  p.l_part = pl.n_splits > 1 ? p.o_part + size_t(pl.n_splits) * size_t(pl.total_rows) * D : nullptr;
  p.q_st = st[0];
  p.k_st = st[1];
  p.v_st = st[2];
  p.o_st = st[3];
  p.total_rows = pl.total_rows;
  p.H = H;
  p.H_kv = H_kv;
  p.group = H / H_kv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.rows = pl.rows;
  p.row_blocks = pl.row_blocks;
  p.n_splits = pl.n_splits;
  p.chunk = pl.chunk;
  p.key_begin = pl.key_begin;
  p.causal = causal;
  p.window = window > Nk ? Nk : window;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.wait_limit_ns = g_wait_limit_ns;
  CUtensorMap tk, tv;
  if (kFp8 ? !make_map_dec_u8(&tk, k, D, Nk, H_kv, B, st[1]) || !make_map_dec_u8(&tv, v, D, Nk, H_kv, B, st[2])
           : !make_map_bf16(&tk, k, D, Nk, H_kv, B, st[1], kDecKeys) ||
                 !make_map_bf16(&tv, v, D, Nk, H_kv, B, st[2], kDecKeys))
    return FA_ERR_CUDA;
  constexpr int smem = DecLayout<D, kFp8>::kSmemBytes;
  if (set_smem(fa_decode_kernel<D, kFp8>, smem) != FA_OK) return FA_ERR_CUDA;
  fa_decode_kernel<D, kFp8><<<unsigned(pl.ctas), kDecThreads, smem, stream>>>(tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (pl.n_splits > 1) {
    const long long blocks = (pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps;
    // programmatic dependent launch: the merge grid is scheduled under the split grid's last
    // wave and waits for its results in the kernel (grid_dep_wait)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(blocks));
    cfg.blockDim = dim3(32 * kDecMergeWarps);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fa_decode_merge_kernel<D>, p) != cudaSuccess) return FA_ERR_CUDA;
    if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

// ---------------------------------------------------------------- backward without caller memory
// Built-in scratch for fa_bwd_noalloc.  It lives in the module's global memory, so every GPU
// that loads this library holds these 64 MiB until the process exits.  Host code must not
// use the array's name as a device address (on the host it is only a stand-in); the device
// address comes from cudaGetSymbolAddress, looked up once per device.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device (nullptr on failure).  Called
// with the device already current; the first call on a device does the lookup.
void* noalloc_scratch(int dev) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

// ---------------------------------------------------------------- self-test kernel
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ alignas(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns);  // nothing ever arrives
  __syncthreads();
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d, const fa_strides* strides,
                    float scale, int causal, int window, void* workspace, size_t workspace_bytes, int phases,
                    void* stream);

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, int window, void* stream) {
  return fa_fwd_gqa(q, k, v, o, lse, B, H, H, N, d, scale, causal, window, stream);
}

int fa_fwd_gqa(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
               int d, float scale, int causal, int window, void* stream) {
  return fa_fwd_strided(q, k, v, o, lse, B, H, H_kv, N, d, nullptr, scale, causal, window, stream);
}

int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N,
                   int d, const fa_strides* strides, float scale, int causal, int window, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  int st = check_problem(B, H, N, d, scale, causal, window);
  if (st == FA_OK) st = check_kv_heads(H, H_kv);
  if (st != FA_OK) return st;
  // q, k, v, o: the caller's strides, or the packed [B, heads, N, d] ones
  Strides s4[4] = {packed(H, N, d), packed(H_kv, N, d), packed(H_kv, N, d), packed(H, N, d)};
  if (strides)
    for (int i = 0; i < 4; ++i) {
      s4[i] = Strides{strides[i].b, strides[i].h, strides[i].n};
      if (!strides_ok(s4[i])) return FA_ERR_ALIGN;
    }
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_fwd<64>(q, k, v, o, lse, B, H, H_kv, N, s4, scale, causal, window, s);
    case 128: return launch_fwd<128>(q, k, v, o, lse, B, H, H_kv, N, s4, scale, causal, window, s);
    default: return launch_fwd256(q, k, v, o, lse, B, H, H_kv, N, s4, scale, causal, window, s);
  }
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_problem(B, H, N, d, 1.f, 0, 0) != FA_OK) return 0;
  return bwd_workspace_bytes((long long)B * H, N, d);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, int window, void* workspace,
           size_t workspace_bytes, void* stream) {
  return fa_bwd_phases(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, window, workspace,
                       workspace_bytes, kBwdAllPhases, stream);
}

int fa_bwd_phases(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                  void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, int window,
                  void* workspace, size_t workspace_bytes, int phases, void* stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, d, nullptr, scale, causal, window, workspace,
                  workspace_bytes, phases, stream);
}

int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
               void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d, float scale, int causal,
               int window, void* workspace, size_t workspace_bytes, int phases, void* stream) {
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, d, nullptr, scale, causal, window, workspace,
                  workspace_bytes, phases, stream);
}

int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d, const fa_strides* strides,
                   float scale, int causal, int window, void* workspace, size_t workspace_bytes, int phases,
                   void* stream) {
  if (!strides) return FA_ERR_NULL;
  return bwd_impl(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, d, strides, scale, causal, window, workspace,
                  workspace_bytes, phases, stream);
}

static int bwd_impl(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                    void* dq, void* dk, void* dv, int B, int H, int H_kv, int N, int d, const fa_strides* strides,
                    float scale, int causal, int window, void* workspace, size_t workspace_bytes, int phases,
                    void* stream) {
  if (phases < 1 || phases > kBwdAllPhases) return FA_ERR_PHASES;
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  int st = check_problem(B, H, N, d, scale, causal, window);
  if (st == FA_OK) st = check_kv_heads(H, H_kv);
  if (st != FA_OK) return st;
  // q, k, v, o, dO, dq, dk, dv: the caller's strides, or the packed ones
  Strides s8[8] = {packed(H, N, d),    packed(H_kv, N, d), packed(H_kv, N, d), packed(H, N, d),
                   packed(H, N, d),    packed(H, N, d),    packed(H_kv, N, d), packed(H_kv, N, d)};
  if (strides)
    for (int i = 0; i < 8; ++i) {
      s8[i] = Strides{strides[i].b, strides[i].h, strides[i].n};
      if (!strides_ok(s8[i])) return FA_ERR_ALIGN;
    }
  const long long BH = (long long)B * H;
  // grid: one CTA per 128-key tile (d = 256: per 64-key tile)
  const long long bwd_ctas = d == 256 ? BH * ((N + kB256Keys - 1) / kB256Keys) : BH * ((N + kBwdKeys - 1) / kBwdKeys);
  if (bwd_ctas > 0x7fffffffLL || BH * padded_rows(N) > 0x7fffffffLL) return FA_ERR_SHAPE;
  if (!workspace || workspace_bytes < bwd_workspace_bytes(BH, N, d)) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) || !aligned(workspace, 16))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, s8, scale, causal, window, workspace, s, phases);
    case 128: return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, s8, scale, causal, window, workspace, s, phases);
    default: return launch_bwd<256>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H_kv, N, s8, scale, causal, window, workspace, s, phases);
  }
}

int fa_fwd_fp8(const void* q8, const void* k8, const void* vt8, float q_scale, float k_scale, float v_scale, void* o,
               float* lse, int B, int H, int H_kv, int N, int d, float scale, int causal, int window, void* stream) {
  if (!q8 || !k8 || !vt8 || !o || !lse) return FA_ERR_NULL;
  int st = check_problem(B, H, N, d, scale, causal, window);
  if (st == FA_OK) st = check_kv_heads(H, H_kv);
  if (st != FA_OK) return st;
  if (d != kF8D) return FA_ERR_HEADDIM;
  if (N % 16) return FA_ERR_SHAPE;   // rows of the transposed V are N bytes: 16-byte multiples
  for (float sc : {q_scale, k_scale, v_scale})
    if (!std::isfinite(sc) || !(sc > 0.f)) return FA_ERR_SCALE;
  if (!aligned(q8, 16) || !aligned(k8, 16) || !aligned(vt8, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  return launch_fwd_fp8(q8, k8, vt8, q_scale, k_scale, v_scale, o, lse, B, H, H_kv, N, scale, causal, window,
                        static_cast<cudaStream_t>(stream));
}

size_t fa_decode_workspace_size(int B, int H, int H_kv, int N_q, int N_k, int d, int causal, int window) {
  DecPlan pl;
  if (check_decode(B, H, H_kv, N_q, N_k, d, 1.f, causal, window, &pl) != FA_OK) return 0;
  return pl.ws_bytes;
}

int fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int H_kv, int N_q,
                  int N_k, int d, const fa_strides* strides, float scale, int causal, int window, void* workspace,
                  size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !lse) return FA_ERR_NULL;
  DecPlan pl;
  int st = check_decode(B, H, H_kv, N_q, N_k, d, scale, causal, window, &pl);
  if (st != FA_OK) return st;
  Strides s4[4] = {packed(H, N_q, d), packed(H_kv, N_k, d), packed(H_kv, N_k, d), packed(H, N_q, d)};
  if (strides)
    for (int i = 0; i < 4; ++i) {
      s4[i] = Strides{strides[i].b, strides[i].h, strides[i].n};
      if (!strides_ok(s4[i])) return FA_ERR_ALIGN;
    }
  if (pl.ws_bytes > 0 && (!workspace || workspace_bytes < pl.ws_bytes)) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 16))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_decode<64, false>(q, k, v, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s);
    case 128: return launch_decode<128, false>(q, k, v, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s);
    default: return launch_decode<256, false>(q, k, v, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s);
  }
}

int fa_fwd_decode_fp8kv(const void* q, const void* k8, const void* v8, float k_scale, float v_scale, void* o,
                        float* lse, int B, int H, int H_kv, int N_q, int N_k, int d, const fa_strides* strides,
                        float scale, int causal, int window, void* workspace, size_t workspace_bytes, void* stream) {
  if (!q || !k8 || !v8 || !o || !lse) return FA_ERR_NULL;
  DecPlan pl;
  int st = check_decode(B, H, H_kv, N_q, N_k, d, scale, causal, window, &pl);
  if (st != FA_OK) return st;
  if (!std::isfinite(k_scale) || !(k_scale > 0.f) || !std::isfinite(v_scale) || !(v_scale > 0.f))
    return FA_ERR_SCALE;
  Strides s4[4] = {packed(H, N_q, d), packed(H_kv, N_k, d), packed(H_kv, N_k, d), packed(H, N_q, d)};
  if (strides)
    for (int i = 0; i < 4; ++i) {
      s4[i] = Strides{strides[i].b, strides[i].h, strides[i].n};
      if (!strides_ok(s4[i])) return FA_ERR_ALIGN;
      // the code arrays are read in 16-byte pieces: 16 one-byte elements
      if ((i == 1 || i == 2) && (s4[i].b % 16 || s4[i].h % 16 || s4[i].n % 16)) return FA_ERR_ALIGN;
    }
  if (pl.ws_bytes > 0 && (!workspace || workspace_bytes < pl.ws_bytes)) return FA_ERR_WORKSPACE;
  if (!aligned(q, 16) || !aligned(k8, 16) || !aligned(v8, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 16))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  switch (d) {
    case 64: return launch_decode<64, true>(q, k8, v8, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s, k_scale, v_scale);
    case 128: return launch_decode<128, true>(q, k8, v8, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s, k_scale, v_scale);
    default: return launch_decode<256, true>(q, k8, v8, o, lse, B, H, H_kv, N_q, N_k, s4, scale, causal, window, workspace, pl, s, k_scale, v_scale);
  }
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_NULL: return "null pointer";
    case FA_ERR_SHAPE: return "bad shape (sizes >= 1, H a multiple of H_kv, N_q <= N_k, within launch limits)";
    case FA_ERR_HEADDIM: return "unsupported head dimension (64, 128 or 256)";
    case FA_ERR_ALIGN: return "misaligned pointer (bf16 arrays 16 B, L 4 B)";
    case FA_ERR_MASK: return "bad mask (causal must be 0 or 1, window >= 0)";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA runtime or launch error";
    case FA_ERR_DEVICE: return "device is not compute capability 10.0 (B200)";
    case FA_ERR_TIMEOUT: return "a kernel-side wait timed out";
    case FA_ERR_SCALE: return "scale must be finite and > 0";
    case FA_ERR_PHASES: return "phase mask must be a non-empty subset of 1 | 2 | 4";
    case FA_ERR_INTERNAL: return "kernel could not run as built (dynamic shared memory not 1 KB aligned)";
    case FA_ERR_NOALLOC_LIMIT: return "problem needs more than the 64 MiB built-in scratch of fa_bwd_noalloc";
    default: return "unknown status";
  }
}

int fa_check_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0 && cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
  if (v & FA_DEVICE_SMEM_ALIGN) return FA_ERR_INTERNAL;
  return v ? FA_ERR_TIMEOUT : FA_OK;
}

void fa_set_wait_limit_ns(unsigned long long limit_ns) {
  g_wait_limit_ns = limit_ns ? limit_ns : kDefaultWaitLimitNs;
}

int fa_selftest_timeout(unsigned long long limit_ns, void* stream) {
  int st = check_device();
  if (st != FA_OK) return st;
  if (limit_ns < 1000ull) limit_ns = 1000ull;
  if (limit_ns > 1000000000ull) limit_ns = 1000000000ull;
  selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, int window,
                   void* stream) {
  if (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv) return FA_ERR_NULL;
  int st = check_problem(B, H, N, d, scale, causal, window);
  if (st != FA_OK) return st;
  const long long BH = (long long)B * H;
  // grid: one CTA per 128-key tile (d = 256: per 64-key tile)
  const long long bwd_ctas = d == 256 ? BH * ((N + kB256Keys - 1) / kB256Keys) : BH * ((N + kBwdKeys - 1) / kBwdKeys);
  if (bwd_ctas > 0x7fffffffLL || BH * padded_rows(N) > 0x7fffffffLL) return FA_ERR_SHAPE;
  if (bwd_workspace_bytes(BH, N, d) > kNoAllocScratchBytes) return FA_ERR_NOALLOC_LIMIT;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGN;
  if ((st = check_device()) != FA_OK) return st;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
  void* ws = noalloc_scratch(dev);
  if (ws == nullptr) return FA_ERR_CUDA;
  // every byte of the scratch the kernels read is rewritten first by fa_bwd_prep (D, L and a
  // zeroed dQ accumulator), so what an earlier call left there does not leak in
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Strides s8[8] = {packed(H, N, d), packed(H, N, d), packed(H, N, d), packed(H, N, d),
                         packed(H, N, d), packed(H, N, d), packed(H, N, d), packed(H, N, d)};
  switch (d) {
    case 64: return launch_bwd<64>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, s8, scale, causal, window, ws, s);
    case 128: return launch_bwd<128>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, s8, scale, causal, window, ws, s);
    default: return launch_bwd<256>(q, k, v, o, lse, dout, dq, dk, dv, B, H, H, N, s8, scale, causal, window, ws, s);
  }
}

}  // extern "C"
