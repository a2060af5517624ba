// Plain fp32-FMA GEMM with the step's epilogues.  It backs the fp32 debug
// precision (no tensor cores, no TF32) and any shape the tensor-core GEMM
// does not take.  C[m,n] = sum_k A(m,k) B(n,k) with either operand stored
// K-major or M/N-major, 64x64 tiles, 256 threads, 4x4 outputs per thread.
#include "common.cuh"
#include "kernels.h"

namespace nc {
namespace {

constexpr int BM = 64, BN = 64, BK = 16;

template <typename T>
__device__ __forceinline__ float ld_op(const T* p, int64_t ld, bool kmajor, int r, int k, int R, int K) {
    if (r >= R || k >= K) return 0.f;
    return tof(kmajor ? p[(int64_t)r * ld + k] : p[(int64_t)k * ld + r]);
}

template <typename T>
__device__ __forceinline__ void st_out(void* C, DType ct, int64_t i, float v) {
    if (ct == DT_BF16) reinterpret_cast<bf16*>(C)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(C)[i] = v;
}

template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmDesc g) {
    __shared__ float As[BK][BM + 4];
    __shared__ float Bs[BK][BN + 4];
    const T* A = reinterpret_cast<const T*>(g.A);
    const T* B = reinterpret_cast<const T*>(g.B);
    int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
    int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < g.K; k0 += BK) {
        for (int i = threadIdx.x; i < BM * BK; i += 256) {
            int r, k;
            if (g.a_kmajor) { r = i / BK; k = i % BK; } else { k = i / BM; r = i % BM; }
            As[k][r] = ld_op(A, g.lda, g.a_kmajor, m0 + r, k0 + k, g.M, g.K);
        }
        for (int i = threadIdx.x; i < BN * BK; i += 256) {
            int r, k;
            if (g.b_kmajor) { r = i / BK; k = i % BK; } else { k = i / BN; r = i % BN; }
            Bs[k][r] = ld_op(B, g.ldb, g.b_kmajor, n0 + r, k0 + k, g.N, g.K);
        }
        __syncthreads();
#pragma unroll
        for (int k = 0; k < BK; ++k) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] = As[k][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; ++j) b[j] = Bs[k][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int m = m0 + ty * 4 + i;
        if (m >= g.M) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int n = n0 + tx * 4 + j;
            if (n >= g.N) continue;
            float v = acc[i][j];
            int64_t ci = (int64_t)m * g.ldc + n;
            switch (g.epi) {
                case EPI_STORE: st_out<T>(g.C, g.c_t, ci, v); break;
                case EPI_ACCUM: reinterpret_cast<float*>(g.C)[ci] += v; break;
                case EPI_RELU2: {
                    float r = fmaxf(v, 0.f);
                    st_out<T>(g.C, g.c_t, ci, r * r);
                    st_out<T>(g.C2, g.c_t, (int64_t)m * g.ldc2 + n, r);
                } break;
                case EPI_RELU2_BWD: {
                    float u = tof(reinterpret_cast<const T*>(g.aux)[(int64_t)m * g.ldaux + n]);
                    st_out<T>(g.C, g.c_t, ci, v * 2.f * u);
                } break;
                case EPI_SOFTCAP: st_out<T>(g.C, g.c_t, ci, g.cap * tanhf(v / g.cap)); break;
            }
        }
    }
}

}  // namespace

cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t s) {
    if (g.M <= 0 || g.N <= 0) return cudaSuccess;
    dim3 grid((g.N + BN - 1) / BN, (g.M + BM - 1) / BM);
    if (grid.y > 65535) return cudaErrorInvalidConfiguration;
    if (g.in_t == DT_BF16) gemm_simt_kernel<bf16><<<grid, 256, 0, s>>>(g);
    else gemm_simt_kernel<float><<<grid, 256, 0, s>>>(g);
    count_launch();
    return cudaGetLastError();
}

}  // namespace nc
