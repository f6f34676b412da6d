// simt_f32.cuh -- fp32 path: the same sharded MLP with fp32 FMA on the CUDA
// cores (no TF32, so the result stays within 1e-5 of the exact block).
// Launch and latency bound at the fp32 block's size (64 x 128 x 512); the
// tensor-core path carries the bf16 workloads.
#pragma once

#include "recipes.cuh"

namespace tspmlp {

// Output tiles are TM x TM (TM = 64: 4 x 4 outputs a thread, for grids that
// fill the part; TM = 16: one output a thread, so a small block still spreads
// over many SMs), with K staged in shared memory KS at a time.
constexpr int kF32TileLarge = 64, kF32KLarge = 16;
constexpr int kF32TileSmall = 16, kF32KSmall = 64;

// H[s*seg_rows + r][j] = act(sum_k X[row][k] * W[k][shard_col(s) + j]) for the
// segment blockIdx.z.
template <int ACT, int TM, int KS>
__global__ void __launch_bounds__(256)
    f32_hidden_kernel(const float* __restrict__ X, const float* __restrict__ Wg,
                      const float* __restrict__ Wu, int d, int f, SegGeom g, int width,
                      float* __restrict__ H, long long ldh) {
    constexpr int RT = TM / 16;  // outputs a thread in each dimension
    __shared__ float xs[KS][TM + 1];
    __shared__ float gs[KS][TM];
    __shared__ float us[KS][TM];
    const int s = blockIdx.z;
    const int r0 = blockIdx.y * TM, c0 = blockIdx.x * TM;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long xrow0 = static_cast<long long>(g.seg_begin + s) * g.seg_rows;
    const int wc0 = g.shard_col(s);
    float ag[RT][RT] = {}, au[RT][RT] = {};
    for (int k0 = 0; k0 < d; k0 += KS) {
        for (int i = threadIdx.x; i < TM * KS; i += 256) {
            const int r = i / KS, kk = i % KS;
            const int rl = r0 + r, k = k0 + kk;
            xs[kk][r] = (rl < g.seg_rows && k < d) ? X[(xrow0 + rl) * d + k] : 0.0f;
        }
        for (int i = threadIdx.x; i < TM * KS; i += 256) {
            const int kk = i / TM, c = i % TM;
            const int cl = c0 + c, k = k0 + kk;
            const bool ok = cl < width && k < d;
            gs[kk][c] = ok ? Wg[static_cast<long long>(k) * f + wc0 + cl] : 0.0f;
            if (ACT == 1) us[kk][c] = ok ? Wu[static_cast<long long>(k) * f + wc0 + cl] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            float a[RT], b[RT], c[RT];
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                a[i] = xs[kk][ty * RT + i];
                b[i] = gs[kk][tx * RT + i];
                c[i] = ACT == 1 ? us[kk][tx * RT + i] : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int j = 0; j < RT; ++j) {
                    ag[i][j] = fmaf(a[i], b[j], ag[i][j]);
                    if (ACT == 1) au[i][j] = fmaf(a[i], c[j], au[i][j]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int rl = r0 + ty * RT + i;
        if (rl >= g.seg_rows) continue;
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const int cl = c0 + tx * RT + j;
            if (cl >= width) continue;
            const float z = ag[i][j];
            const float h = ACT == 1 ? (z / (1.0f + expf(-z))) * au[i][j]
                                     : 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
            H[static_cast<long long>(s * g.seg_rows + rl) * ldh + cl] = h;
        }
    }
}

// Y[row][c] (first ? = : +=) sum_j H[s*seg_rows + r][j] * Wd[shard_col(s) + j][c]
// -- the chunk's partial output (its shards in order along K) added into the
// fp32 output in place.
template <int TM, int KS>
__global__ void __launch_bounds__(256)
    f32_down_kernel(const float* __restrict__ H, long long ldh, const float* __restrict__ Wd, int d,
                    SegGeom g, int width, int first, float* __restrict__ Y) {
    constexpr int RT = TM / 16;
    __shared__ float hs[KS][TM + 1];
    __shared__ float ws[KS][TM];
    const int s = blockIdx.z;
    const int r0 = blockIdx.y * TM, c0 = blockIdx.x * TM;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const long long hrow0 = static_cast<long long>(s) * g.seg_rows;
    const long long yrow0 = static_cast<long long>(g.seg_begin + s) * g.seg_rows;
    const int wr0 = g.shard_col(s);
    float acc[RT][RT] = {};
    for (int k0 = 0; k0 < width; k0 += KS) {
        for (int i = threadIdx.x; i < TM * KS; i += 256) {
            const int r = i / KS, kk = i % KS;
            const int rl = r0 + r, k = k0 + kk;
            hs[kk][r] = (rl < g.seg_rows && k < width) ? H[(hrow0 + rl) * ldh + k] : 0.0f;
        }
        for (int i = threadIdx.x; i < TM * KS; i += 256) {
            const int kk = i / TM, c = i % TM;
            const int cl = c0 + c, k = k0 + kk;
            ws[kk][c] = (cl < d && k < width) ? Wd[static_cast<long long>(wr0 + k) * d + cl] : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
            float a[RT], b[RT];
#pragma unroll
            for (int i = 0; i < RT; ++i) {
                a[i] = hs[kk][ty * RT + i];
                b[i] = ws[kk][tx * RT + i];
            }
#pragma unroll
            for (int i = 0; i < RT; ++i)
#pragma unroll
                for (int j = 0; j < RT; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < RT; ++i) {
        const int rl = r0 + ty * RT + i;
        if (rl >= g.seg_rows) continue;
#pragma unroll
        for (int j = 0; j < RT; ++j) {
            const int cl = c0 + tx * RT + j;
            if (cl >= d) continue;
            float* y = Y + (yrow0 + rl) * d + cl;
            *y = first ? acc[i][j] : *y + acc[i][j];
        }
    }
}

}  // namespace tspmlp
