// BF16 GEMM C = A * W^T (f32 out) with warp-level mma.sync m16n8k16.
// A [M, K] bf16 (activations, row stride lda), W [N, K] bf16 (weights,
// row-major), both K-contiguous.  128x128x32 block tile, 8 warps of 64x32,
// 3-stage cp.async pipeline, XOR-swizzled shared memory for conflict-free
// ldmatrix.  This is the portable baseline used for prefill projections.
#include "common.cuh"

namespace dory {

namespace {

constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// Byte offset of 16-byte chunk c (0..3) of row r inside a [rows][32] bf16
// tile (64 B per row), swizzled so 8 consecutive rows hit distinct banks.
__device__ __forceinline__ int swz(int r, int c) {
  return r * 64 + ((c ^ ((r >> 1) & 3)) << 4);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src,
                                           int bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst),
               "l"(src), "r"(bytes));
}

__global__ void __launch_bounds__(256)
gemm_mma_kernel(const bf16* __restrict__ A, int lda,
                const bf16* __restrict__ W, float* __restrict__ C, int ldc,
                int M, int N, int K, const float* __restrict__ col_scale) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sA = smem;                          // STAGES x BM x 64 B
  uint8_t* sB = smem + STAGES * BM * 64;       // STAGES x BN x 64 B
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  const int KT = K / BK;
  pdl_wait();
  pdl_trigger();

  auto load_stage = [&](int s, int kt) {
    const int k0 = kt * BK;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int id = tid + i * 256;
      const int r = id >> 2, c = id & 3;
      const int gm = m0 + r;
      const bf16* src = A + (size_t)(gm < M ? gm : 0) * lda + k0 + c * 8;
      cp_async16(smem_u32(sA + s * BM * 64 + swz(r, c)), src, gm < M ? 16 : 0);
      const bf16* srcb = W + (size_t)(n0 + r) * K + k0 + c * 8;
      cp_async16(smem_u32(sB + s * BN * 64 + swz(r, c)), srcb, 16);
    }
  };

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[i][j][k] = 0.f;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < KT) load_stage(s, s);
    asm volatile("cp.async.commit_group;\n" ::);
  }

  for (int kt = 0; kt < KT; ++kt) {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(STAGES - 2));
    __syncthreads();
    const int nk = kt + STAGES - 1;
    if (nk < KT) load_stage(nk % STAGES, nk);
    asm volatile("cp.async.commit_group;\n" ::);

    const uint8_t* tA = sA + (kt % STAGES) * BM * 64;
    const uint8_t* tB = sB + (kt % STAGES) * BN * 64;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {          // two k16 steps per BK = 32
      uint32_t af[4][4], bfr[4][2];
#pragma unroll
      for (int mi = 0; mi < 4; ++mi) {
        const int r = wm * 64 + mi * 16 + (lane & 15);
        const int c = kk * 2 + (lane >> 4);
        asm volatile(
            "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
            : "=r"(af[mi][0]), "=r"(af[mi][1]), "=r"(af[mi][2]), "=r"(af[mi][3])
            : "r"(smem_u32(tA + swz(r, c))));
      }
#pragma unroll
      for (int nj = 0; nj < 2; ++nj) {
        const int r = wn * 32 + nj * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int c = kk * 2 + ((lane >> 3) & 1);
        uint32_t t0, t1, t2, t3;
        asm volatile(
            "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
            : "=r"(t0), "=r"(t1), "=r"(t2), "=r"(t3)
            : "r"(smem_u32(tB + swz(r, c))));
        bfr[nj * 2][0] = t0; bfr[nj * 2][1] = t1;
        bfr[nj * 2 + 1][0] = t2; bfr[nj * 2 + 1][1] = t3;
      }
#pragma unroll
      for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 4; ++ni)
          asm volatile(
              "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
              "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
              : "+f"(acc[mi][ni][0]), "+f"(acc[mi][ni][1]),
                "+f"(acc[mi][ni][2]), "+f"(acc[mi][ni][3])
              : "r"(af[mi][0]), "r"(af[mi][1]), "r"(af[mi][2]), "r"(af[mi][3]),
                "r"(bfr[ni][0]), "r"(bfr[ni][1]));
    }
  }
  asm volatile("cp.async.wait_group 0;\n" ::);

#pragma unroll
  for (int mi = 0; mi < 4; ++mi) {
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int col = n0 + wn * 32 + ni * 8 + (lane & 3) * 2;
      const float s0 = col_scale ? col_scale[col] : 1.f;
      const float s1 = col_scale ? col_scale[col + 1] : 1.f;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = m0 + wm * 64 + mi * 16 + (lane >> 2) + h * 8;
        if (row < M) {
          float2 v = make_float2(acc[mi][ni][2 * h] * s0, acc[mi][ni][2 * h + 1] * s1);
          *reinterpret_cast<float2*>(C + (size_t)row * ldc + col) = v;
        }
      }
    }
  }
}

}  // namespace

void launch_gemm_bf16(const bf16* A, int lda, const bf16* W, float* C, int ldc,
                      int M, int N, int K, const float* col_scale,
                      cudaStream_t st) {
  const size_t smem = (size_t)STAGES * (BM + BN) * 64;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(gemm_mma_kernel,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = true;
  }
  dim3 grid(N / BN, (M + BM - 1) / BM);
  launch_k(gemm_mma_kernel, grid, dim3(256), smem, st, A, lda, W, C, ldc, M,
           N, K, col_scale);
}

}  // namespace dory
