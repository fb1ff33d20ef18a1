// Test-only: launches a kernel of the host emulation (cuda_emu.h) over its
// grid, one block after another, as stream order allows.  Every block's
// dynamic shared memory is allocated to its exact size and filled with NaN
// bytes, so AddressSanitizer sees accesses past it and values read before
// they were written show up.  Launch<Args>(kernel, grid, shared bytes, args)
// returns false where a CUDA launch would fail on the shared-memory size.
#ifndef SSD_EMU_LAUNCH_H_
#define SSD_EMU_LAUNCH_H_

#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

#include "cuda_emu.h"

namespace emu {

inline constexpr int kThreads = 256;              // threads per block of every kernel here
inline constexpr size_t kEmuSmemLimit = 232448;   // dynamic shared memory one CTA may opt into on sm_100

#ifdef SSD_EMU_THREADS
// Each block: kThreads host threads meeting at a std::barrier.
template <class Args>
struct Launch {
  int launches = 0;
  bool reverse = false;  // (thread order only matters for fibers)
  bool operator()(void (*kern)(Args), unsigned grid, size_t smem, const Args& k) {
    if (smem > kEmuSmemLimit) return false;
    ++launches;
    gridDim = dim3{grid, 1, 1};
    blockDim = dim3{(unsigned)kThreads, 1, 1};
    for (unsigned bi = 0; bi < grid; ++bi) {
      void* sm = smem ? std::malloc(smem) : nullptr;
      if (sm) std::memset(sm, 0xff, smem);
      std::barrier<> bar(kThreads);
      emu::g_barrier = &bar;
      emu::g_smem = static_cast<float*>(sm);
      std::vector<std::thread> th;
      th.reserve(kThreads);
      for (int t = 0; t < kThreads; ++t) {
        th.emplace_back([&bar, kern, &k, bi, t] {
          threadIdx = dim3{(unsigned)t, 1, 1};
          blockIdx = dim3{bi, 1, 1};
          kern(k);
          bar.arrive_and_drop();  // an exited thread no longer holds back __syncthreads
        });
      }
      for (auto& x : th) x.join();
      std::free(sm);
    }
    return true;
  }
  bool record(void*) { return true; }  // no events on the host
};
#else
// Each block: kThreads fibers on this host thread.  A round resumes every
// live fiber once, in thread order (or reversed), and each runs up to its
// next __syncthreads or its end; so no fiber starts phase k+1 before all
// have finished phase k, as a CTA barrier guarantees, and a value read
// across threads without a barrier between is seen unwritten (NaN) in one
// of the two orders.
inline constexpr size_t kFiberStack = 256 * 1024;
inline std::vector<char> g_done;
inline int g_cur = 0;
inline void (*g_entry)() = nullptr;  // runs the kernel on the running fiber

inline void fiber_entry() {
  g_entry();
  g_done[g_cur] = 1;  // returning resumes the scheduler (uc_link)
}

template <class Args>
struct Bound {  // the kernel and arguments the fibers of a launch run
  static inline void (*kern)(Args) = nullptr;
  static inline const Args* args = nullptr;
  static void run() { kern(*args); }
};

template <class Args>
struct Launch {
  int launches = 0;
  bool reverse = false;
  std::vector<ucontext_t> ctx;
  std::vector<char*> stacks;
  ~Launch() {
    for (char* p : stacks) std::free(p);
  }
  bool operator()(void (*kern)(Args), unsigned grid, size_t smem, const Args& k) {
    if (smem > kEmuSmemLimit) return false;
    ++launches;
    if (stacks.empty()) {
      ctx.resize(kThreads);
      for (int t = 0; t < kThreads; ++t) stacks.push_back(static_cast<char*>(std::malloc(kFiberStack)));
    }
    gridDim = dim3{grid, 1, 1};
    blockDim = dim3{(unsigned)kThreads, 1, 1};
    Bound<Args>::kern = kern;
    Bound<Args>::args = &k;
    g_entry = &Bound<Args>::run;
    g_done.assign(kThreads, 0);
    for (unsigned bi = 0; bi < grid; ++bi) {
      void* sm = smem ? std::malloc(smem) : nullptr;
      if (sm) std::memset(sm, 0xff, smem);
      emu::g_smem = static_cast<float*>(sm);
      blockIdx = dim3{bi, 1, 1};
      for (int t = 0; t < kThreads; ++t) {
        getcontext(&ctx[t]);
        ctx[t].uc_stack.ss_sp = stacks[t];
        ctx[t].uc_stack.ss_size = kFiberStack;
        ctx[t].uc_link = &emu::g_sched;
        makecontext(&ctx[t], fiber_entry, 0);
        g_done[t] = 0;
      }
      int live = kThreads;
      while (live > 0) {
        for (int j = 0; j < kThreads; ++j) {
          const int t = reverse ? kThreads - 1 - j : j;
          if (g_done[t]) continue;
          threadIdx = dim3{(unsigned)t, 1, 1};
          g_cur = t;
          emu::g_self = &ctx[t];
          swapcontext(&emu::g_sched, &ctx[t]);
          if (g_done[t]) --live;
        }
      }
      std::free(sm);
    }
    return true;
  }
  bool record(void*) { return true; }  // no events on the host
};
#endif

}  // namespace emu

#endif  // SSD_EMU_LAUNCH_H_
