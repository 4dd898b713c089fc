// gdn_state.cu -- state algebra for sharding one sequence over segments.
//
// Over a segment of tokens the recurrence S_t = S_{t-1} A_t + beta_t v_t k_t^T,
// A_t = Diag(alpha_t)(I - beta_t k_t k_t^T) (FG2-GDN section 1; GDN's scalar
// alpha_t is the special case), is affine in the state it starts from:
//   S_end = S_start M + B,   M = A_1 ... A_n (d_k x d_k),  B = S_end from S = 0.
// B is the prefill's final state from a zero state; M is its final state from the
// identity with V = 0 (every row of the state is a probe vector).  Chaining
// segments composes these maps, S_start(r + 1) = S_start(r) M_r + B_r, so the
// segments of one long sequence can run on different GPUs and exchange only the
// maps.  This file holds the two small kernels of that exchange:
//   compose:  out = s m + b   per (sequence, head), fp32, d_v x d_k times d_k x d_k;
//   identity: out = I         per (sequence, head) (d_v = d_k).
// It also holds FG2-GDN+'s value scaling, v~ = sqrt(beta^v) . v (section 3.4 of
// the FG2-GDN page), written once before the prefill reads v~ in place of v.
#include <algorithm>

#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kTile = 32;  // output tile 32 x 32, k-steps of 32; 32 x 8 threads

// One block per (output tile, sequence-head), blockIdx.x = tile + tiles * (n H + h),
// tiles = (d_v / 32) (d_k / 32): thread (tx, ty) computes rows
// ty, ty + 8, ty + 16, ty + 24 of column tx of the tile.  out may alias b (each
// element of b is read once, by the thread that writes it), not s or m.
__global__ void __launch_bounds__(256)
compose_kernel(const float *s, const float *m, const float *b, float *out, int dv, int dk) {
    __shared__ float ts[kTile][kTile + 1];
    __shared__ float tm[kTile][kTile + 1];
    const int ct = dk / kTile, tiles = ct * (dv / kTile);
    const long long nh = blockIdx.x / tiles;
    const int tile = (int)(blockIdx.x % tiles);
    const int row0 = (tile / ct) * kTile, col0 = (tile % ct) * kTile;
    const int tx = threadIdx.x, ty = threadIdx.y;
    const float *sp = s + (size_t)nh * dv * dk;
    const float *mp = m + (size_t)nh * dk * dk;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k0 = 0; k0 < dk; k0 += kTile) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ty + 8 * i;
            ts[r][tx] = sp[(size_t)(row0 + r) * dk + k0 + tx];
            tm[r][tx] = mp[(size_t)(k0 + r) * dk + col0 + tx];
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < kTile; ++kk) {
            const float mv = tm[kk][tx];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[i] = fmaf(ts[ty + 8 * i][kk], mv, acc[i]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const size_t o = (size_t)nh * dv * dk + (size_t)(row0 + ty + 8 * i) * dk + col0 + tx;
        out[o] = acc[i] + (b ? b[o] : 0.f);
    }
}

// FG2-GDN+'s scaled values, 8 elements per step: 16 bytes of v, 32 of rates.
__global__ void value_rate_kernel(const uint4 *v, const float4 *bv, uint4 *out, long long n8) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n8;
         i += (long long)gridDim.x * blockDim.x) {
        const uint4 x = v[i];
        const float4 b0 = bv[2 * i], b1 = bv[2 * i + 1];
        const float r[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float lo = __uint_as_float(w[j] << 16) * sqrtf(r[2 * j]);
            const float hi = __uint_as_float(w[j] & 0xffff0000u) * sqrtf(r[2 * j + 1]);
            __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
            y[j] = *reinterpret_cast<uint32_t *>(&t);
        }
        out[i] = make_uint4(y[0], y[1], y[2], y[3]);
    }
}

__global__ void identity_kernel(float *out, int d, long long total) {
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const long long e = i % ((long long)d * d);
        out[i] = (e / d == e % d) ? 1.f : 0.f;
    }
}

}  // namespace

cudaError_t launch_state_compose(const float *s, const float *m, const float *b, float *out,
                                 long long nh, int dv, int dk, cudaStream_t st, int *launches) {
    if (nh == 0) return cudaSuccess;
    const long long blocks = nh * (dk / kTile) * (dv / kTile);
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    compose_kernel<<<(unsigned)blocks, dim3(kTile, 8), 0, st>>>(s, m, b, out, dv, dk);
    if (launches) ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_value_rate(const void *v, const float *beta_v, void *out, long long n,
                              cudaStream_t st, int *launches) {
    if (n == 0) return cudaSuccess;
    if (n % 8) return cudaErrorInvalidValue;
    const long long n8 = n / 8;
    const long long blocks = std::min<long long>((n8 + 255) / 256, 148LL * 32);
    value_rate_kernel<<<(unsigned)blocks, 256, 0, st>>>(reinterpret_cast<const uint4 *>(v),
                                                         reinterpret_cast<const float4 *>(beta_v),
                                                         reinterpret_cast<uint4 *>(out), n8);
    if (launches) ++*launches;
    return cudaGetLastError();
}

cudaError_t launch_state_identity(float *out, long long nh, int d, cudaStream_t st, int *launches) {
    const long long total = nh * d * d;
    if (total == 0) return cudaSuccess;
    const long long blocks = std::min<long long>((total + 255) / 256, 148LL * 16);
    identity_kernel<<<(unsigned)blocks, 256, 0, st>>>(out, d, total);
    if (launches) ++*launches;
    return cudaGetLastError();
}

}  // namespace gdn
