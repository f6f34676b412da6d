// simt_f32.cuh -- fp32 path: the same sharded MLP with fp32 FMA on the CUDA
// cores (no TF32, so the result stays within 1e-5 of the exact block).
// Launch and latency bound at the fp32 block's size (64 x 128 x 512); the
// tensor-core path carries the bf16 workloads.
#pragma once

#include "recipes.cuh"

namespace tspmlp {

constexpr int kF32Tile = 64;  // output tile edge
constexpr int kF32K = 16;     // K step staged in shared memory

// H[s*seg_rows + r][j] = act(sum_k X[row][k] * W[k][shard_col(s) + j]) for the
// segment blockIdx.z; 4 x 4 outputs a thread.
template <int ACT>
__global__ void __launch_bounds__(256)
    f32_hidden_kernel(const float* __restrict__ X, const float* __restrict__ Wg,
                      const float* __restrict__ Wu, int d, int f, SegGeom g, int width,
                      float* __restrict__ H, long long ldh) {
    __shared__ float xs[kF32K][kF32Tile + 1];
    __shared__ float gs[kF32K][kF32Tile];
    __shared__ float us[kF32K][kF32Tile];
    const int s = blockIdx.z;
    const int r0 = blockIdx.y * kF32Tile, c0 = blockIdx.x * kF32Tile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long xrow0 = static_cast<long long>(g.seg_begin + s) * g.seg_rows;
    const int wc0 = g.shard_col(s);
    float ag[4][4] = {}, au[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += kF32K) {
        for (int i = threadIdx.x; i < kF32Tile * kF32K; i += 256) {
            const int r = i / kF32K, kk = i % kF32K;
            const int rl = r0 + r, k = k0 + kk;
            xs[kk][r] = (rl < g.seg_rows && k < d) ? X[(xrow0 + rl) * d + k] : 0.0f;
        }
        for (int i = threadIdx.x; i < kF32Tile * kF32K; i += 256) {
            const int kk = i / kF32Tile, c = i % kF32Tile;
            const int cl = c0 + c, k = k0 + kk;
            const bool ok = cl < width && k < d;
            gs[kk][c] = ok ? Wg[static_cast<long long>(k) * f + wc0 + cl] : 0.0f;
            if (ACT == 1) us[kk][c] = ok ? Wu[static_cast<long long>(k) * f + wc0 + cl] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kF32K; ++kk) {
            float a[4], b[4], c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = xs[kk][ty * 4 + i];
                b[i] = gs[kk][tx * 4 + i];
                c[i] = ACT == 1 ? us[kk][tx * 4 + i] : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    ag[i][j] = fmaf(a[i], b[j], ag[i][j]);
                    if (ACT == 1) au[i][j] = fmaf(a[i], c[j], au[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rl = r0 + ty * 4 + i;
        if (rl >= g.seg_rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cl = c0 + tx * 4 + j;
            if (cl >= width) continue;
            const float z = ag[i][j];
            const float h = ACT == 1 ? (z / (1.0f + expf(-z))) * au[i][j]
                                     : 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
            H[static_cast<long long>(s * g.seg_rows + rl) * ldh + cl] = h;
        }
    }
}

// Y[row][c] (first ? = : +=) sum_j H[s*seg_rows + r][j] * Wd[shard_col(s) + j][c]
// -- the shard's partial output added into the fp32 output in place.
__global__ void __launch_bounds__(256)
    f32_down_kernel(const float* __restrict__ H, long long ldh, const float* __restrict__ Wd, int d,
                    SegGeom g, int width, int first, float* __restrict__ Y) {
    __shared__ float hs[kF32K][kF32Tile + 1];
    __shared__ float ws[kF32K][kF32Tile];
    const int s = blockIdx.z;
    const int r0 = blockIdx.y * kF32Tile, c0 = blockIdx.x * kF32Tile;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long hrow0 = static_cast<long long>(s) * g.seg_rows;
    const long long yrow0 = static_cast<long long>(g.seg_begin + s) * g.seg_rows;
    const int wr0 = g.shard_col(s);
    float acc[4][4] = {};
    for (int k0 = 0; k0 < width; k0 += kF32K) {
        for (int i = threadIdx.x; i < kF32Tile * kF32K; i += 256) {
            const int r = i / kF32K, kk = i % kF32K;
            const int rl = r0 + r, k = k0 + kk;
            hs[kk][r] = (rl < g.seg_rows && k < width) ? H[(hrow0 + rl) * ldh + k] : 0.0f;
        }
        for (int i = threadIdx.x; i < kF32Tile * kF32K; i += 256) {
            const int kk = i / kF32Tile, c = i % kF32Tile;
            const int cl = c0 + c, k = k0 + kk;
            ws[kk][c] = (cl < d && k < width) ? Wd[static_cast<long long>(wr0 + k) * d + cl] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kF32K; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = hs[kk][ty * 4 + i];
                b[i] = ws[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int rl = r0 + ty * 4 + i;
        if (rl >= g.seg_rows) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int cl = c0 + tx * 4 + j;
            if (cl >= d) continue;
            float* y = Y + (yrow0 + rl) * d + cl;
            *y = first ? acc[i][j] : *y + acc[i][j];
        }
    }
}

}  // namespace tspmlp
