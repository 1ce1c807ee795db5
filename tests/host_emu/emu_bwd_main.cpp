// TEST INFRASTRUCTURE ONLY: runs the backward of bwd_kernel.cuh (fa_bwd_prep, fa_bwd_kernel<EMU_D>,
// fa_bwd_dq_final) on the host through the emulation of emu.h / sm100_stub.cuh, with the tensor
// maps, workspace and parameters the library derives for packed [B, heads, N, d] arrays.
// usage: emu_bwd_main B H Hkv N causal window scale prefix
//   reads prefix.q .k .v .o .do (bf16) and .lse (fp32); writes prefix.dq .dk .dv (bf16)
#include "emu.h"
#ifdef EMU_BWD256
#include "bwd256_kernel.cuh"
#define EMU_D 256
#else
#include "bwd_kernel.cuh"
#endif

#include <fstream>
#include <string>

#ifndef EMU_D
#define EMU_D 128
#endif

namespace fa {
#ifdef EMU_BWD256
alignas(1024) uint8_t smem_raw[sizeof(Bwd256Smem)];
#else
alignas(1024) uint8_t smem_raw[sizeof(BwdSmem<EMU_D>)];
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

int main(int argc, char** argv) {
  if (argc != 9) { std::fprintf(stderr, "bad args\n"); return 2; }
  const int B = atoi(argv[1]), H = atoi(argv[2]), Hkv = atoi(argv[3]), N = atoi(argv[4]), causal = atoi(argv[5]),
            window = atoi(argv[6]);
  const float scale = float(atof(argv[7]));
  const std::string prefix = argv[8];
  constexpr int D = EMU_D;
  const size_t nq = size_t(B) * H * N * D, nkv = size_t(B) * Hkv * N * D;
  auto q = read_file<uint16_t>(prefix + ".q", nq);
  auto k = read_file<uint16_t>(prefix + ".k", nkv);
  auto v = read_file<uint16_t>(prefix + ".v", nkv);
  auto o = read_file<uint16_t>(prefix + ".o", nq);
  auto dout = read_file<uint16_t>(prefix + ".do", nq);
  auto lse = read_file<float>(prefix + ".lse", size_t(B) * H * N);
  std::vector<uint16_t> dq(nq, 0x7fc0), dk(nkv, 0x7fc0), dv(nkv, 0x7fc0);
  const int BH = B * H, BH_kv = B * Hkv;
  const int Np = (N + kBwdRows - 1) / kBwdRows * kBwdRows;
  std::vector<float> ws(size_t(BH) * Np * (2 + D), NAN);
  float* lp = ws.data();
  float* dd = lp + size_t(BH) * Np;
  float* dq_acc = dd + size_t(BH) * Np;
  const Strides st_q{(long long)H * N * D, (long long)N * D, (long long)D};
  const Strides st_kv{(long long)Hkv * N * D, (long long)N * D, (long long)D};
  constexpr int G = D / 8;
  const long long prep_rows = (long long)BH * Np;
  emu_launch(unsigned((prep_rows + (256 / G) - 1) / (256 / G)), 256, 0, [&] {
    fa_bwd_prep<D>(reinterpret_cast<const __nv_bfloat16*>(o.data()), reinterpret_cast<const __nv_bfloat16*>(dout.data()),
                   lse.data(), lp, dd, dq_acc, N, Np, H, st_q, st_q, prep_rows);
  });
#ifdef EMU_BWD256
  constexpr int box_keys = kB256Keys;
#else
  constexpr int box_keys = kBwdKeys;
#endif
  const CUtensorMap tq = make_map(q.data(), D, N, H, B, kBwdRows), tk = make_map(k.data(), D, N, Hkv, B, box_keys),
                    tv = make_map(v.data(), D, N, Hkv, B, box_keys), tdo = make_map(dout.data(), D, N, H, B, kBwdRows);
  // the fp32 dQ accumulator [BH, Np, D] as (D, Np, BH, 1), 32 x 32 boxes
  CUtensorMap tdq;
  tdq.base = reinterpret_cast<const unsigned char*>(dq_acc);
  tdq.dims[0] = uint64_t(D);
  tdq.dims[1] = uint64_t(Np);
  tdq.dims[2] = uint64_t(BH);
  tdq.dims[3] = 1;
  tdq.strides[0] = uint64_t(D) * 4;
  tdq.strides[1] = uint64_t(Np) * D * 4;
  tdq.strides[2] = uint64_t(BH) * Np * D * 4;
  tdq.box_x = 32;
  tdq.box_rows = 32;
  tdq.esize = 4;
  // dK and dV as (D, N, H_kv, B), 32-row boxes (the backward's TMA-store epilogue)
  const CUtensorMap tdk = make_map(dk.data(), D, N, Hkv, B, 32), tdv = make_map(dv.data(), D, N, Hkv, B, 32);
  BwdParams prm;
  prm.lp = lp;
  prm.dd = dd;
  prm.dq_acc = dq_acc;
  prm.dk = reinterpret_cast<__nv_bfloat16*>(dk.data());
  prm.dv = reinterpret_cast<__nv_bfloat16*>(dv.data());
  prm.N = N;
  prm.Np = Np;
  prm.BH = BH;
  prm.H = H;
  prm.H_kv = Hkv;
  prm.group = H / Hkv;
  prm.dk_st = st_kv;
  prm.dv_st = st_kv;
  prm.n_kv_tiles = (N + box_keys - 1) / box_keys;
  prm.causal = causal;
  prm.window = window > N ? N : window;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.scale = scale;
  prm.wait_limit_ns = 60ull * 1000000000ull;
#ifdef EMU_BWD256
  emu_launch(unsigned(prm.n_kv_tiles) * unsigned(BH_kv), kB256Threads, sizeof(fa::smem_raw),
             [&] { fa_bwd256_kernel(tq, tk, tv, tdo, tdq, prm); }, fa::smem_raw);
#else
  // the form the host library launches: dK from the shared-memory dS when K/V heads are shared
  if (prm.group > 1)
    emu_launch(unsigned(prm.n_kv_tiles) * unsigned(BH_kv), kBwdThreads, sizeof(fa::smem_raw),
               [&] { fa_bwd_kernel<D, true>(tq, tk, tv, tdo, tdq, tdk, tdv, prm); }, fa::smem_raw);
  else
    emu_launch(unsigned(prm.n_kv_tiles) * unsigned(BH_kv), kBwdThreads, sizeof(fa::smem_raw),
               [&] { fa_bwd_kernel<D, false>(tq, tk, tv, tdo, tdq, tdk, tdv, prm); }, fa::smem_raw);
#endif
  if (g_status != 0) { std::fprintf(stderr, "device status %d\n", g_status); return 3; }
  const long long rows = (long long)BH * N;
  emu_launch(unsigned((rows + (256 / G) - 1) / (256 / G)), 256, 0, [&] {
    fa_bwd_dq_final<D>(dq_acc, reinterpret_cast<__nv_bfloat16*>(dq.data()), N, Np, scale, H, st_q, rows);
  });
  write_file(prefix + ".dq", dq);
  write_file(prefix + ".dk", dk);
  write_file(prefix + ".dv", dv);
  return 0;
}
