// TEST INFRASTRUCTURE ONLY: runs fa_fwd_kernel<EMU_D> of fwd_kernel.cuh (or, with EMU_FWD256,
// fa_fwd256_kernel of fwd256_kernel.cuh) on the host through the emulation of emu.h /
// sm100_stub.cuh, with the tensor maps and parameters the library derives for packed
// [B, heads, N, d] arrays.
// usage: emu_fwd_main B H Hkv N causal window scale prefix   (prefix.q/.k/.v bf16; writes .o, .lse)
#include "emu.h"
#if defined(EMU_FWD256)
#include "fwd256_kernel.cuh"
#define EMU_D 256
#elif defined(EMU_FWD_FP8)
#include "fwd_fp8_kernel.cuh"
#define EMU_D 128
#else
#include "fwd_kernel.cuh"
#endif

#include <fstream>
#include <string>

#ifndef EMU_D
#define EMU_D 128
#endif

namespace fa {
// the kernel's dynamic shared memory: exactly one (1024-byte aligned) FwdSmem, so AddressSanitizer
// sees any access past it
#if defined(EMU_FWD256)
alignas(1024) uint8_t smem_raw[sizeof(Fwd256Smem)];
#elif defined(EMU_FWD_FP8)
alignas(1024) uint8_t smem_raw[sizeof(FwdFp8Smem)];
#else
alignas(1024) uint8_t smem_raw[sizeof(FwdSmem<EMU_D>)];
#endif
}  // namespace fa

using namespace fa;

template <class T>
std::vector<T> read_file(const std::string& path, size_t n) {
  std::vector<T> v(n);
  std::ifstream f(path, std::ios::binary);
  f.read(reinterpret_cast<char*>(v.data()), n * sizeof(T));
  if (!f) { std::fprintf(stderr, "short read %s\n", path.c_str()); std::exit(2); }
  return v;
}
template <class T>
void write_file(const std::string& path, const std::vector<T>& v) {
  std::ofstream f(path, std::ios::binary);
  f.write(reinterpret_cast<const char*>(v.data()), v.size() * sizeof(T));
}

CUtensorMap make_map(const uint16_t* base, int d, int rows, int heads, int B, int box_rows) {
  CUtensorMap m;
  m.base = reinterpret_cast<const unsigned char*>(base);
  m.dims[0] = uint64_t(d);
  m.dims[1] = uint64_t(rows);
  m.dims[2] = uint64_t(heads);
  m.dims[3] = uint64_t(B);
  m.strides[0] = uint64_t(d) * 2;
  m.strides[1] = uint64_t(rows) * d * 2;
  m.strides[2] = uint64_t(heads) * rows * d * 2;
  m.box_x = 64;
  m.box_rows = uint32_t(box_rows);
  return m;
}

#ifdef EMU_FWD_FP8
// E4M3 code arrays: q8, k8 [B, heads, N, 128]; vt8 [B, H_kv, 128, N]
// usage: emu_fwd_fp8 B H Hkv N causal window scale prefix s_q s_k s_v
int main(int argc, char** argv) {
  if (argc != 12) { std::fprintf(stderr, "bad args\n"); return 2; }
  const int B = atoi(argv[1]), H = atoi(argv[2]), Hkv = atoi(argv[3]), N = atoi(argv[4]), causal = atoi(argv[5]),
            window = atoi(argv[6]);
  const float scale = float(atof(argv[7]));
  const std::string prefix = argv[8];
  const float s_q = float(atof(argv[9])), s_k = float(atof(argv[10])), s_v = float(atof(argv[11]));
  constexpr int D = 128;
  auto q = read_file<uint8_t>(prefix + ".q", size_t(B) * H * N * D);
  auto k = read_file<uint8_t>(prefix + ".k", size_t(B) * Hkv * N * D);
  auto vt = read_file<uint8_t>(prefix + ".v", size_t(B) * Hkv * D * N);
  std::vector<uint16_t> o(size_t(B) * H * N * D, 0x7fc0);
  std::vector<float> lse(size_t(B) * H * N, NAN);
  auto map8 = [](const uint8_t* base, uint64_t x, uint64_t rows, uint64_t heads, uint64_t b) {
    CUtensorMap m;
    m.base = base;
    m.dims[0] = x;
    m.dims[1] = rows;
    m.dims[2] = heads;
    m.dims[3] = b;
    m.strides[0] = x;
    m.strides[1] = rows * x;
    m.strides[2] = heads * rows * x;
    m.box_x = 128;
    m.box_rows = 128;
    m.esize = 1;
    return m;
  };
  const CUtensorMap tq = map8(q.data(), D, N, H, B), tk = map8(k.data(), D, N, Hkv, B),
                    tvt = map8(vt.data(), N, D, Hkv, B);
  FwdParams prm;
  prm.o = reinterpret_cast<__nv_bfloat16*>(o.data());
  prm.lse = lse.data();
  prm.N = N;
  prm.BH = B * H;
  prm.H = H;
  prm.group = H / Hkv;
  prm.o_st = Strides{(long long)H * N * D, (long long)N * D, (long long)D};
  prm.n_pairs = ((N + kBlockM - 1) / kBlockM + kQTiles - 1) / kQTiles;
  prm.causal = causal;
  prm.window = window > N ? N : window;
  prm.scale_log2 = scale * s_q * s_k * 1.4426950408889634f;
  prm.wait_limit_ns = 60ull * 1000000000ull;
  const unsigned grid = unsigned(prm.n_pairs) * unsigned(B * H);
  emu_launch(grid, kFwdThreads, sizeof(fa::smem_raw), [&] { fa_fwd_fp8_kernel(tq, tk, tvt, prm, s_v); }, fa::smem_raw);
  if (g_status != 0) { std::fprintf(stderr, "device status %d\n", g_status); return 3; }
  write_file(prefix + ".o", o);
  write_file(prefix + ".lse", lse);
  return 0;
}
#else
int main(int argc, char** argv) {
  if (argc != 9) { std::fprintf(stderr, "bad args\n"); return 2; }
  const int B = atoi(argv[1]), H = atoi(argv[2]), Hkv = atoi(argv[3]), N = atoi(argv[4]), causal = atoi(argv[5]),
            window = atoi(argv[6]);
  const float scale = float(atof(argv[7]));
  const std::string prefix = argv[8];
  constexpr int D = EMU_D;
  auto q = read_file<uint16_t>(prefix + ".q", size_t(B) * H * N * D);
  auto k = read_file<uint16_t>(prefix + ".k", size_t(B) * Hkv * N * D);
  auto v = read_file<uint16_t>(prefix + ".v", size_t(B) * Hkv * N * D);
  std::vector<uint16_t> o(size_t(B) * H * N * D, 0x7fc0);
  std::vector<float> lse(size_t(B) * H * N, NAN);
#ifdef EMU_FWD256
  constexpr int box_q = k256BlockM, box_kv = k256BlockN;
#else
  constexpr int box_q = kBlockM, box_kv = kBlockN;
#endif
  const CUtensorMap tq = make_map(q.data(), D, N, H, B, box_q), tk = make_map(k.data(), D, N, Hkv, B, box_kv),
                    tv = make_map(v.data(), D, N, Hkv, B, box_kv);
  FwdParams prm;
  prm.o = reinterpret_cast<__nv_bfloat16*>(o.data());
  prm.lse = lse.data();
  prm.N = N;
  prm.BH = B * H;
  prm.H = H;
  prm.group = H / Hkv;
  prm.o_st = Strides{(long long)H * N * D, (long long)N * D, (long long)D};
#ifdef EMU_FWD256
  prm.n_pairs = (N + k256BlockM - 1) / k256BlockM;   // query tiles per head
#else
  prm.n_pairs = ((N + kBlockM - 1) / kBlockM + kQTiles - 1) / kQTiles;
#endif
  prm.causal = causal;
  prm.window = window > N ? N : window;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = 60ull * 1000000000ull;
  const unsigned grid = unsigned(prm.n_pairs) * unsigned(B * H);
  std::printf("grid %u smem %zu\n", grid, sizeof(fa::smem_raw));
#if defined(EMU_FWD256)
  emu_launch(grid, k256Threads, sizeof(fa::smem_raw), [&] { fa_fwd256_kernel(tq, tk, tv, prm); }, fa::smem_raw);
#else
  const CUtensorMap to = make_map(o.data(), D, N, H, B, box_q);
  emu_launch(grid, kFwdThreads, sizeof(fa::smem_raw), [&] { fa_fwd_kernel<D>(tq, tk, tv, to, prm); }, fa::smem_raw);
#endif
  if (g_status != 0) { std::fprintf(stderr, "device status %d\n", g_status); return 3; }
  write_file(prefix + ".o", o);
  write_file(prefix + ".lse", lse);
  return 0;
}
#endif
