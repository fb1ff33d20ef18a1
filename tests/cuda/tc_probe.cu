// Test-only probe of the tcgen05 building blocks used by the fused SSD kernel:
// one CTA computes D = A B^T (A: M x K, B: N x K, bf16, row-major in global
// memory) with the shared-memory layouts, descriptors, MMA shapes and TMEM
// load shapes of each step of that kernel, and writes D (M x N, fp32) back in
// logical order.  The tests compare D with a float64 matmul.
//
// mode 0: M=64,  N=64, K=128  A K-major (2 x 64-wide K blocks), B K-major      (C B^T)
// mode 1: M=64,  N=64, K=64   A K-major,                        B MN-major     (W X)
// mode 2: M=64,  N=64, K=128  A K-major (2 K blocks),           B MN-major     (C H^T)
// mode 3: M=128, N=64, K=64   A MN-major (2 x 64-wide M blocks), B MN-major    (B^T X~)
// mode 4: M=128, N=64, K=64   A MN-major (2 x 64-wide M blocks), B K-major     (X'^T W'^T)
// mode 5: M=128, N=64, K=128  A in TMEM (32x32b stores),         B K-major     (H C^T)
// mode 6: M=128, N=64, K=64   A in TMEM: MN-major smem tile moved by 8 x 8
//                             transposes and 16x128b stores,      B MN-major    (X'^T B)
// modes 0-2 read TMEM with the 16-lane x2 shape, modes 3 and 5 with 32x32b,
// modes 4 and 6 with 16x256b.
//
// tc_probe_layout records the lane / column maps of the 16x256b load, the
// 16x128b store and the 8 x 8 transpose, so the tests can check them exactly.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "sm100.cuh"

using namespace ssd::sm100;

namespace {


__global__ void __launch_bounds__(128) probe_kernel(int mode, const __nv_bfloat16* __restrict__ A,
                                                    const __nv_bfloat16* __restrict__ B, float* __restrict__ D,
                                                    int* __restrict__ err) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // 1024-align the dynamic smem base
  unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* sA = smem;                 // 32 KB
  unsigned char* sB = smem + 32768;         // 16 KB
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  int M = 64, N = 64, K = 128;
  if (mode == 1) K = 64;
  if (mode == 3 || mode == 4 || mode == 6) { M = 128; K = 64; }
  if (mode == 5) M = 128;

  // ---- stage A and B in shared memory with the kernel's layouts
  for (int i = tid; i < M * K; i += 128) {
    const int m = i / K, k = i % K;
    const __nv_bfloat16 v = A[m * K + k];
    uint32_t off;
    if (mode == 5) break;  // written straight to TMEM below
    if (mode == 3 || mode == 4 || mode == 6) {  // MN-major: blocks of 64 m, rows = k, 128 B per row
      off = (m / 64) * 8192 + k * 128 + (m % 64) * 2;
    } else {          // K-major: blocks of 64 k, rows = m, 128 B per row
      off = (k / 64) * 8192 + m * 128 + (k % 64) * 2;
    }
    *reinterpret_cast<__nv_bfloat16*>(sA + sw128(off)) = v;
  }
  for (int i = tid; i < N * K; i += 128) {
    const int n = i / K, k = i % K;
    const __nv_bfloat16 v = B[n * K + k];
    uint32_t off;
    if (mode == 0 || mode == 4 || mode == 5) {  // K-major: blocks of 64 k, rows = n
      off = (k / 64) * 8192 + n * 128 + (k % 64) * 2;
    } else {          // MN-major: rows = k, 64 n per row
      off = k * 128 + n * 2;
    }
    *reinterpret_cast<__nv_bfloat16*>(sB + sw128(off)) = v;
  }
  if (tid == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  fence_proxy_async_smem();
  __syncthreads();
  if (warp == 0) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // A operand in TMEM columns 64.. (modes 5, 6)
  if (mode == 5) {
    const int m = 32 * warp + lane;
    for (int half = 0; half < 2; ++half) {
      uint32_t r[32];
      for (int c = 0; c < 32; ++c) {
        const int k = 2 * (32 * half + c);
        const __nv_bfloat162 v = __halves2bfloat162(A[m * K + k], A[m * K + k + 1]);
        r[c] = *reinterpret_cast<const uint32_t*>(&v);
      }
      SSD_TMEM_ST_32x32b_X32(tmem + ((uint32_t)(32 * warp) << 16) + 64 + 32 * half, r);
    }
  } else if (mode == 6) {
    for (int mh = 0; mh < 32; mh += 16)
      for (int kg = 0; kg < 64; kg += 32) {
        uint32_t r[8];
        for (int j = 0; j < 4; ++j)
          for (int e = 0; e < 2; ++e) {
            const int m = 32 * warp + mh + 8 * e + 2 * (lane % 4), k = kg + 8 * j + lane / 4;
            const uint32_t off = (m / 64) * 8192 + k * 128 + (m % 64) * 2;
            r[2 * j + e] = movmatrix_trans(*reinterpret_cast<const uint32_t*>(sA + sw128(off)));
          }
        SSD_TMEM_ST_16x128b_X4(tmem + ((uint32_t)(32 * warp + mh) << 16) + 64 + kg / 2, r);
      }
  }
  tmem_wait_st();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (tid == 0) {
    const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB);
    for (int kk = 0; kk < K / 16; ++kk) {
      uint64_t ad, bd;
      uint32_t id;
      if (mode == 5 || mode == 6) {
        bd = mode == 5 ? sw128_desc(b0 + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024)
                       : sw128_desc(b0 + kk * 16 * 128, 8192, 1024);
        mma_bf16_ts(tmem, tmem + 64 + kk * 8, bd, idesc_bf16(128, 64, 0, mode == 6), kk > 0 ? 1u : 0u);
        continue;
      }
      if (mode == 3 || mode == 4) {
        ad = sw128_desc(a0 + kk * 16 * 128, 8192, 1024);
        bd = mode == 3 ? sw128_desc(b0 + kk * 16 * 128, 8192, 1024) : sw128_desc(b0 + kk * 32, 16, 1024);
        id = idesc_bf16(128, 64, 1, mode == 3);
      } else {
        ad = sw128_desc(a0 + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024);
        if (mode == 0) {
          bd = sw128_desc(b0 + (kk / 4) * 8192 + (kk % 4) * 32, 16, 1024);
          id = idesc_bf16(64, 64, 0, 0);
        } else {
          bd = sw128_desc(b0 + kk * 16 * 128, 8192, 1024);
          id = idesc_bf16(64, 64, 0, 1);
        }
      }
      mma_bf16_ss(tmem, ad, bd, id, kk > 0 ? 1u : 0u);
    }
    mma_commit(&bar);
  }
  __syncwarp();
  const bool ok = mbar_wait(&bar, 0, &abort_flag, 1000000000ull);
  tc_fence_after();
  if (!ok) {
    if (tid == 0) *err = 1;
  } else {
    const int q = warp;  // TMEM lane quadrant of this warp
    uint32_t r[32];
    if (mode == 4 || mode == 6) {
      for (int lh = 0; lh < 32; lh += 16)
        for (int ch = 0; ch < 64; ch += 32) {
          SSD_TMEM_LD_16x256b_X4(tmem + ((uint32_t)(32 * q + lh) << 16) + ch, r);
          SSD_TMEM_WAIT_LD_16(r);
          for (int j = 0; j < 4; ++j)
            for (int e = 0; e < 4; ++e) {
              const int m = 32 * q + lh + lane / 4 + 8 * (e >> 1), n = ch + 8 * j + 2 * (lane % 4) + (e & 1);
              D[m * N + n] = __uint_as_float(r[4 * j + e]);
            }
        }
    } else if (mode == 3 || mode == 5) {
      for (int half = 0; half < 2; ++half) {
        SSD_TMEM_LD_32x32b_X32(tmem + ((uint32_t)(32 * q) << 16) + half * 32, r);
        SSD_TMEM_WAIT_LD_32(r);
        const int m = 32 * q + lane;
        for (int j = 0; j < 32; ++j) D[m * N + half * 32 + j] = __uint_as_float(r[j]);
      }
    } else {
      SSD_TMEM_LD_16x32bx2_X32_HALF32(tmem + ((uint32_t)(32 * q) << 16), r);
      SSD_TMEM_WAIT_LD_32(r);
      const int m = 16 * q + (lane % 16);
      const int n0 = (lane / 16) * 32;
      for (int j = 0; j < 32; ++j) D[m * N + n0 + j] = __uint_as_float(r[j]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

// out[0, 2048): thread t, register j of a 16x256b.x4 load at lanes 32(t/32)..,
//   columns 0.., after columns 0..63 were filled with (lane << 16) | column
// out[2048, 4096): lane l, column c of columns 64..79 read with 32x32b after a
//   16x128b.x4 store of ((thread << 8) | register) at lanes 32(l/32)..
//   (columns never stored keep 0xffffffff)
// out[4096, 4128): 8 x 8 transpose of thread i's (row i/4, columns 2(i%4),
//   2(i%4)+1), with element ids row * 8 + column
// out[4128, 4256): ldmatrix.x4.trans, thread i register k, from four 8 x 8
//   matrices in shared memory holding ids 64 k + 8 row + column
// out[4256, 4384): the shared memory written by stmatrix.x4.trans of
//   fragments holding ids 64 k + 8 (i/4) + 2(i%4) (+1), as 16-bit pairs
__global__ void __launch_bounds__(128) layout_kernel(uint32_t* __restrict__ out) {
  __shared__ uint32_t tmem_base;
  __shared__ __align__(16) uint16_t mats[2][256];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  if (warp == 0) {
    tmem_alloc(&tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base, tq = tmem + ((uint32_t)(32 * warp) << 16);
  uint32_t r[32];
  for (int half = 0; half < 2; ++half) {
    for (int c = 0; c < 32; ++c) r[c] = ((uint32_t)tid << 16) | (uint32_t)(32 * half + c);
    SSD_TMEM_ST_32x32b_X32(tq + 32 * half, r);
  }
  for (int c = 0; c < 32; ++c) r[c] = 0xffffffffu;
  SSD_TMEM_ST_32x32b_X32(tq + 64, r);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  tc_fence_after();
  SSD_TMEM_LD_16x256b_X4(tq, r);
  SSD_TMEM_WAIT_LD_16(r);
  for (int j = 0; j < 16; ++j) out[tid * 16 + j] = r[j];
  for (int j = 0; j < 8; ++j) r[j] = ((uint32_t)tid << 8) | (uint32_t)j;
  SSD_TMEM_ST_16x128b_X4(tq + 64, r);
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  tc_fence_after();
  SSD_TMEM_LD_32x32b_X16(tq + 64, r);
  SSD_TMEM_WAIT_LD_16(r);
  for (int j = 0; j < 16; ++j) out[2048 + tid * 16 + j] = r[j];
  if (warp == 0) {
    const uint32_t lo = (uint32_t)((lane / 4) * 8 + 2 * (lane % 4));
    out[4096 + lane] = movmatrix_trans(lo | ((lo + 1) << 16));
    for (int e = lane; e < 256; e += 32) mats[0][e] = (uint16_t)e;
    __syncwarp();
    uint32_t v[4];
    ldmatrix_x4_trans(smem_u32(&mats[0][(lane / 8) * 64 + (lane % 8) * 8]), v);
    for (int k = 0; k < 4; ++k) {
      out[4128 + lane * 4 + k] = v[k];
      const uint32_t id = (uint32_t)(64 * k + 8 * (lane / 4) + 2 * (lane % 4));
      v[k] = id | ((id + 1) << 16);
    }
    stmatrix_x4_trans(smem_u32(&mats[1][(lane / 8) * 64 + (lane % 8) * 8]), v);
    __syncwarp();
    for (int e = lane; e < 128; e += 32) out[4256 + e] = reinterpret_cast<const uint32_t*>(mats[1])[e];
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace

extern "C" __attribute__((visibility("default"))) int tc_probe_mma(int mode, const void* A, const void* B,
                                                                   float* D, int* err, void* stream) {
  if (mode < 0 || mode > 6) return 1;
  const size_t smem = 32768 + 16384 + 1024;
  if (cudaFuncSetAttribute(probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return 2;
  probe_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      mode, static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), D, err);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

extern "C" __attribute__((visibility("default"))) int tc_probe_layout(uint32_t* out, void* stream) {
  layout_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(out);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}

