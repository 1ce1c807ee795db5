// TEST INFRASTRUCTURE ONLY: runs the decode kernels of decode_kernel.cuh on the host through
// the SIMT emulation of emu.h, with the launch parameters fa_fwd_decode derives.
// usage: emu_main B H Hkv Nq Nk d causal window scale  sq(3) sk(3) sv(3) so(3)  nq nk nv no  prefix
//                 [k_scale v_scale]   (with the scales: prefix.k / prefix.v hold E4M3 codes, one byte each)
#include "emu.h"
#include "decode_kernel.cuh"

#include <fstream>
#include <string>

using namespace fa;

// the kernels' dynamic shared memory, on a 1 KB boundary as on the device (the swizzled ring
// stages are placed relative to it)
alignas(1024) static unsigned char dec_smem[232448];

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

int main(int argc, char** argv) {
  const int base_args = 1 + 9 + 12 + 4 + 1;
  if (argc != base_args && argc != base_args + 2) { std::fprintf(stderr, "bad args\n"); return 2; }
  const bool fp8 = argc == base_args + 2;
  int a = 1;
  const int B = atoi(argv[a++]), H = atoi(argv[a++]), Hkv = atoi(argv[a++]), Nq = atoi(argv[a++]),
            Nk = atoi(argv[a++]), d = atoi(argv[a++]), causal = atoi(argv[a++]), window = atoi(argv[a++]);
  const float scale = float(atof(argv[a++]));
  Strides st[4];
  for (int i = 0; i < 4; ++i) {
    st[i].b = atoll(argv[a++]);
    st[i].h = atoll(argv[a++]);
    st[i].n = atoll(argv[a++]);
  }
  size_t n[4];
  for (int i = 0; i < 4; ++i) n[i] = size_t(atoll(argv[a++]));
  const std::string prefix = argv[a++];
  const float k_scale = fp8 ? float(atof(argv[a++])) : 1.f, v_scale = fp8 ? float(atof(argv[a++])) : 1.f;
  auto q = read_file<uint16_t>(prefix + ".q", n[0]);
  std::vector<uint16_t> k, v;
  std::vector<uint8_t> k8, v8;
  if (fp8) {
    k8 = read_file<uint8_t>(prefix + ".k", n[1]);
    v8 = read_file<uint8_t>(prefix + ".v", n[2]);
  } else {
    k = read_file<uint16_t>(prefix + ".k", n[1]);
    v = read_file<uint16_t>(prefix + ".v", n[2]);
  }
  std::vector<uint16_t> o(n[3], 0x7fc0);   // NaN: rows the kernels fail to write show up
  std::vector<float> lse(size_t(B) * H * Nq, NAN);

  const int win = window > Nk ? Nk : window;
  const DecPlan pl = dec_plan(B, H, Hkv, Nq, Nk, d, causal, win);
  std::vector<float> ws(pl.ws_bytes / 4 + 1, NAN);
  DecParams p;
  p.q = reinterpret_cast<const __nv_bfloat16*>(q.data());
  p.v_scale = v_scale;
  p.o = reinterpret_cast<__nv_bfloat16*>(o.data());
  p.lse = lse.data();
  p.o_part = pl.ws_bytes ? ws.data() : nullptr;
  p.l_part = pl.n_splits > 1 ? p.o_part + size_t(pl.n_splits) * size_t(pl.total_rows) * d : nullptr;
  p.q_st = st[0];
  p.k_st = st[1];
  p.v_st = st[2];
  p.o_st = st[3];
  p.total_rows = pl.total_rows;
  p.H = H;
  p.H_kv = Hkv;
  p.group = H / Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.rows = pl.rows;
  p.row_blocks = pl.row_blocks;
  p.n_splits = pl.n_splits;
  p.chunk = pl.chunk;
  p.key_begin = pl.key_begin;
  p.causal = causal;
  p.window = win;
  p.scale_log2 = scale * k_scale * 1.4426950408889634f;
  p.wait_limit_ns = 2000000000ull;
  // K and V as the tensor maps fa_fwd_decode encodes: (d, N_k, H_kv, B), 16-row boxes of 64 bf16
  // or 128 codes (128-byte swizzled), at d = 64 with E4M3 codes 64 unswizzled
  auto kv_map = [&](const void* base, const Strides& s) {
    CUtensorMap m;
    const uint32_t es = fp8 ? 1 : 2;
    m.base = static_cast<const unsigned char*>(base);
    m.dims[0] = uint64_t(d);
    m.dims[1] = uint64_t(Nk);
    m.dims[2] = uint64_t(Hkv);
    m.dims[3] = uint64_t(B);
    m.strides[0] = uint64_t(s.n) * es;
    m.strides[1] = uint64_t(s.h) * es;
    m.strides[2] = uint64_t(s.b) * es;
    m.box_x = fp8 && d >= 128 ? 128 : 64;
    m.box_rows = kDecKeys;
    m.esize = es;
    m.swizzle = fp8 && d < 128 ? 0 : 128;
    return m;
  };
  const CUtensorMap tk = fp8 ? kv_map(k8.data(), st[1]) : kv_map(k.data(), st[1]);
  const CUtensorMap tv = fp8 ? kv_map(v8.data(), st[2]) : kv_map(v.data(), st[2]);
  std::printf("plan rows=%d row_blocks=%d n_splits=%d chunk=%d key_begin=%d ctas=%lld ws=%zu\n", pl.rows,
              pl.row_blocks, pl.n_splits, pl.chunk, pl.key_begin, pl.ctas, pl.ws_bytes);
  if (d == 256) {
    if (fp8)
      emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<256, true>::kSmemBytes, [&] { fa_decode_kernel<256, true>(tk, tv, p); }, dec_smem);
    else
      emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<256>::kSmemBytes, [&] { fa_decode_kernel<256, false>(tk, tv, p); }, dec_smem);
    if (pl.n_splits > 1)
      emu_launch(unsigned((pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps), 32 * kDecMergeWarps, 0,
                 [&] { fa_decode_merge_kernel<256>(p); });
  } else if (fp8 && d == 64) {
    emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<64, true>::kSmemBytes, [&] { fa_decode_kernel<64, true>(tk, tv, p); }, dec_smem);
    if (pl.n_splits > 1)
      emu_launch(unsigned((pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps), 32 * kDecMergeWarps, 0,
                 [&] { fa_decode_merge_kernel<64>(p); });
  } else if (fp8) {
    emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<128, true>::kSmemBytes,
               [&] { fa_decode_kernel<128, true>(tk, tv, p); }, dec_smem);
    if (pl.n_splits > 1)
      emu_launch(unsigned((pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps), 32 * kDecMergeWarps, 0,
                 [&] { fa_decode_merge_kernel<128>(p); });
  } else if (d == 64) {
    emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<64>::kSmemBytes, [&] { fa_decode_kernel<64, false>(tk, tv, p); }, dec_smem);
    if (pl.n_splits > 1)
      emu_launch(unsigned((pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps), 32 * kDecMergeWarps, 0,
                 [&] { fa_decode_merge_kernel<64>(p); });
  } else {
    emu_launch(unsigned(pl.ctas), kDecThreads, DecLayout<128>::kSmemBytes, [&] { fa_decode_kernel<128, false>(tk, tv, p); }, dec_smem);
    if (pl.n_splits > 1)
      emu_launch(unsigned((pl.total_rows + kDecMergeWarps - 1) / kDecMergeWarps), 32 * kDecMergeWarps, 0,
                 [&] { fa_decode_merge_kernel<128>(p); });
  }
  write_file(prefix + ".o", o);
  write_file(prefix + ".lse", lse);
  return 0;
}
