// Test-only driver: runs ssd_bwd's host plan and kernels (ssd_bwd.cuh) on the
// CPU through the emulation in cuda_emu.h.  Blocks and kernels run one after
// another, as stream order allows.
//
//   bwd_emu DIR
//
// reads DIR/args.txt ("key value" lines: the size fields of ssd_bwd_args,
// dtype 0|1 and has_* / want_* flags) and the input arrays DIR/<name>.bin
// (raw, row-major: x dt A B C D h0 seq dy dfinal z), writes the gradients as
// raw fp32 to DIR/<name>.bin (dx ddt dA dB dC dD dh0 dz) and prints the status.
// "reverse 1" runs each block's fibers in reverse thread order; "flags" are
// ssd_bwd_args.flags (with SSD_BWD_DINITIAL_ONLY only dh0 is allocated).
// Every buffer is allocated to its exact size, so AddressSanitizer sees any
// access past it; outputs, workspace and shared memory start as NaN bytes,
// so a value read before it was written shows up in the result.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <string>
#include <thread>
#include <vector>

#include "cuda_emu.h"
#include "emu_launch.h"
#include "ssd.h"
#include "ssd_bwd.cuh"

namespace {

struct Buf {
  void* p = nullptr;
  size_t n = 0;
};

Buf read_file(const std::string& path) {
  Buf b;
  FILE* f = std::fopen(path.c_str(), "rb");
  if (!f) return b;
  std::fseek(f, 0, SEEK_END);
  b.n = (size_t)std::ftell(f);
  std::fseek(f, 0, SEEK_SET);
  b.p = std::malloc(b.n ? b.n : 1);
  if (std::fread(b.p, 1, b.n, f) != b.n) std::abort();
  std::fclose(f);
  return b;
}

void write_file(const std::string& path, const void* p, size_t n) {
  FILE* f = std::fopen(path.c_str(), "wb");
  if (!f || std::fwrite(p, 1, n, f) != n) std::abort();
  std::fclose(f);
}

float* nan_floats(size_t n) {
  float* p = static_cast<float*>(std::malloc(n * 4));
  std::memset(p, 0xff, n * 4);
  return p;
}

static_assert(emu::kThreads == ssd::bwd::kThreads, "the emulator launches the kernels' block size");
using EmuLaunch = emu::Launch<ssd::bwd::KArgs>;

}  // namespace

int main(int argc, char** argv) {
  if (argc != 2) {
    std::fprintf(stderr, "usage: bwd_emu DIR\n");
    return 2;
  }
  const std::string dir = argv[1];
  std::map<std::string, long long> kv;
  {
    FILE* f = std::fopen((dir + "/args.txt").c_str(), "r");
    if (!f) return 2;
    char key[64];
    long long v;
    while (std::fscanf(f, "%63s %lld", key, &v) == 2) kv[key] = v;
    std::fclose(f);
  }
  ssd_bwd_args a;
  std::memset(&a, 0, sizeof(a));
  a.batch = kv["batch"];
  a.seqlen = kv["seqlen"];
  a.nheads = kv["nheads"];
  a.headdim = kv["headdim"];
  a.dstate = kv["dstate"];
  a.ngroups = kv["ngroups"];
  a.chunk_size = kv["chunk_size"];
  a.dtype = (ssd_dtype)kv["dtype"];
  a.flags = (uint32_t)kv["flags"];
  const bool only_dh0 = (a.flags & SSD_BWD_DINITIAL_ONLY) != 0;
  auto in = [&](const char* name, bool present) -> const void* {
    if (!present) return nullptr;
    Buf b = read_file(dir + "/" + name + ".bin");
    if (!b.p) {
      std::fprintf(stderr, "missing %s\n", name);
      std::exit(2);
    }
    return b.p;
  };
  a.x = in("x", true);
  a.dt = static_cast<const float*>(in("dt", true));
  a.A = static_cast<const float*>(in("A", true));
  a.B = in("B", true);
  a.C = in("C", true);
  a.D = static_cast<const float*>(in("D", kv["has_D"] != 0));
  a.initial_states = static_cast<const float*>(in("h0", kv["has_h0"] != 0));
  a.seq_idx = static_cast<const int32_t*>(in("seq", kv["has_seq"] != 0));
  a.dy = in("dy", true);
  a.dfinal_states = static_cast<const float*>(in("dfinal", kv["has_dfinal"] != 0));
  a.z = in("z", kv["has_z"] != 0);

  const size_t b = a.batch, L = a.seqlen, H = a.nheads, P = a.headdim, N = a.dstate, G = a.ngroups;
  const size_t nx = b * L * H * P, ndt = b * L * H, nB = b * L * G * N, nh = b * H * P * N;
  if (!only_dh0) {
    a.dx = nan_floats(nx);
    a.ddt = nan_floats(ndt);
    a.dA = nan_floats(H);
    a.dB = nan_floats(nB);
    a.dC = nan_floats(nB);
    a.dD = kv["want_dD"] ? nan_floats(H) : nullptr;
    a.dz = a.z ? nan_floats(nx) : nullptr;
  }
  a.dinitial_states = kv["want_dh0"] ? nan_floats(nh) : nullptr;

  ssd::bwd::Plan pl;
  ssd_status st = ssd::bwd::plan(&a, &pl);
  void* ws = nullptr;
  if (st == SSD_OK) {
    ws = std::aligned_alloc(256, pl.total ? pl.total : 256);
    std::memset(ws, 0xff, pl.total);
    a.workspace = ws;
    a.workspace_bytes = pl.total;
  }
  EmuLaunch launch;
  launch.reverse = kv["reverse"] != 0;
  st = ssd::bwd::run(&a, launch);
  std::printf("status %d launches %d chunk %lld\n", (int)st, launch.launches, (long long)pl.d.Q);
  if (st != SSD_OK) return 1;
  if (a.dx) write_file(dir + "/dx.bin", a.dx, nx * 4);
  if (a.ddt) write_file(dir + "/ddt.bin", a.ddt, ndt * 4);
  if (a.dA) write_file(dir + "/dA.bin", a.dA, H * 4);
  if (a.dB) write_file(dir + "/dB.bin", a.dB, nB * 4);
  if (a.dC) write_file(dir + "/dC.bin", a.dC, nB * 4);
  if (a.dD) write_file(dir + "/dD.bin", a.dD, H * 4);
  if (a.dinitial_states) write_file(dir + "/dh0.bin", a.dinitial_states, nh * 4);
  if (a.dz) write_file(dir + "/dz.bin", a.dz, nx * 4);
  std::free(ws);
  return 0;
}
