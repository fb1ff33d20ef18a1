// Test-only driver: runs ssd_conv1d_silu_bwd's plan and kernels
// (ssd_conv_bwd.cuh) on the CPU through the emulation in cuda_emu.h.
//
//   conv_bwd_emu DIR
//
// reads DIR/args.txt ("key value" lines: batch seqlen channels width dtype
// has_bias has_seq want_dbias reverse) and the raw inputs DIR/<name>.bin
// (u w bias seq dout), writes du, dw, dbias as raw fp32 and prints the
// status.  Buffers are allocated to their exact sizes and outputs and
// workspace start as NaN bytes, as in bwd_emu.cpp.
#include <cstdio>
#include <cstdlib>
#include <map>
#include <string>

#include "cuda_emu.h"
#include "emu_launch.h"
#include "ssd.h"
#include "ssd_conv_bwd.cuh"

static_assert(emu::kThreads == ssd::convbwd::kThreads, "the emulator launches the kernels' block size");

namespace {

void* read_file(const std::string& path) {
  FILE* f = std::fopen(path.c_str(), "rb");
  if (!f) {
    std::fprintf(stderr, "missing %s\n", path.c_str());
    std::exit(2);
  }
  std::fseek(f, 0, SEEK_END);
  const size_t n = (size_t)std::ftell(f);
  std::fseek(f, 0, SEEK_SET);
  void* p = std::malloc(n ? n : 1);
  if (std::fread(p, 1, n, f) != n) std::abort();
  std::fclose(f);
  return p;
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

}  // namespace

int main(int argc, char** argv) {
  if (argc != 2) return 2;
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
  ssd_conv_bwd_args a;
  std::memset(&a, 0, sizeof(a));
  a.batch = kv["batch"];
  a.seqlen = kv["seqlen"];
  a.channels = kv["channels"];
  a.width = kv["width"];
  a.dtype = (ssd_dtype)kv["dtype"];
  a.u = read_file(dir + "/u.bin");
  a.weight = static_cast<const float*>(read_file(dir + "/w.bin"));
  a.bias = kv["has_bias"] ? static_cast<const float*>(read_file(dir + "/bias.bin")) : nullptr;
  a.seq_idx = kv["has_seq"] ? static_cast<const int32_t*>(read_file(dir + "/seq.bin")) : nullptr;
  a.dout = read_file(dir + "/dout.bin");
  const size_t n = (size_t)(a.batch * a.seqlen * a.channels), C = (size_t)a.channels, K = (size_t)a.width;
  a.du = nan_floats(n);
  a.dweight = nan_floats(C * K);
  a.dbias = kv["want_dbias"] ? nan_floats(C) : nullptr;
  const size_t ws = ssd_conv1d_silu_bwd_workspace_size(&a);
  if (ws) {
    a.workspace = std::aligned_alloc(256, ws);
    std::memset(a.workspace, 0xff, ws);
    a.workspace_bytes = ws;
  }
  emu::Launch<ssd::convbwd::KArgs> launch;
  launch.reverse = kv["reverse"] != 0;
  const ssd_status st = ssd::convbwd::run(&a, launch);
  std::printf("status %d launches %d\n", (int)st, launch.launches);
  if (st != SSD_OK) return 1;
  write_file(dir + "/du.bin", a.du, n * 4);
  write_file(dir + "/dw.bin", a.dweight, C * K * 4);
  if (a.dbias) write_file(dir + "/dbias.bin", a.dbias, C * 4);
  return 0;
}

// the workspace query, as libssd exports it
extern "C" size_t ssd_conv1d_silu_bwd_workspace_size(const ssd_conv_bwd_args* a) {
  ssd::convbwd::KArgs k;
  size_t ws = 0;
  return ssd::convbwd::plan(a, &k, &ws) == SSD_OK ? ws : 0;
}
