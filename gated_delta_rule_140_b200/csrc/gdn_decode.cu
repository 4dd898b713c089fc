// gdn_decode.cu -- one recurrent decode step, state updated in place.
//
// For every (sequence, head) and every state row i (output channel), with
// S_i the row of the fp32 state [d_v][d_k]:
//   GDN:  r = S_i.k, s = S_i.q, delta_i = beta (v_i - alpha r),
//         o_i = alpha s + delta_i (k.q),   S_i <- alpha S_i + delta_i k
//   KDA:  S~_i = S_i . alpha (per key channel), r = S~_i.k, s = S~_i.q,
//         delta_i = beta (v_i - r), o_i = s + delta_i (k.q), S_i <- S~_i + delta_i k
// which is S <- S Diag(alpha)(I - beta k k^T) + beta v k^T, o = S q (FG2-GDN
// section 1; the decode step keeps a constant-size state per head).
//
// The step is pure HBM streaming (64 KiB read + 64 KiB written per head for
// d = 128, against ~0.5 KiB of token data), so the kernel is laid out for
// bandwidth: a warp owns whole rows, each lane holds DK/32 consecutive
// columns (one 16-byte float4 for d_k = 128), ROWS rows are loaded before any
// reduction so every lane keeps ROWS independent 16-byte loads in flight, the
// two dot products are reduced together with warp shuffles, and the row is
// written back in place with one vector store per lane.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kWarps = 4;
constexpr int kRows = 4;  // rows in flight per warp

template <int VEC>
struct VecF;
template <>
struct VecF<4> {
    using T = float4;
};
template <>
struct VecF<2> {
    using T = float2;
};

__device__ __forceinline__ void load_vec(const void *p, long long i, int bf16, float *x, int n) {
    if (bf16) {
        const __nv_bfloat16 *b = reinterpret_cast<const __nv_bfloat16 *>(p) + i;
        if (n == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(b);
            const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&u.x);
            const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&u.y);
            x[0] = __low2float(lo); x[1] = __high2float(lo);
            x[2] = __low2float(hi); x[3] = __high2float(hi);
        } else {
            const __nv_bfloat162 u = *reinterpret_cast<const __nv_bfloat162 *>(b);
            x[0] = __low2float(u); x[1] = __high2float(u);
        }
    } else {
        const float *f = reinterpret_cast<const float *>(p) + i;
        for (int j = 0; j < n; ++j) x[j] = f[j];
    }
}

template <int DK, bool CH>
__global__ void __launch_bounds__(kWarps * 32)
decode_kernel(DecodeArgs a) {
    constexpr int VEC = DK / 32;
    using V = typename VecF<VEC>::T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nh = blockIdx.x;  // n * H + h
    const int dv = a.dv;

    float kk[VEC], qq[VEC], al[VEC];
    load_vec(a.k, (long long)nh * DK + lane * VEC, a.bf16, kk, VEC);
    load_vec(a.q, (long long)nh * DK + lane * VEC, a.bf16, qq, VEC);
    const float beta = a.beta[nh];
    if (CH) {
#pragma unroll
        for (int j = 0; j < VEC; ++j) al[j] = expf(a.log_alpha[(long long)nh * DK + lane * VEC + j]);
    } else {
        const float alpha = expf(a.log_alpha[nh]);
#pragma unroll
        for (int j = 0; j < VEC; ++j) al[j] = alpha;
    }
    float kq = 0.f;
#pragma unroll
    for (int j = 0; j < VEC; ++j) kq += kk[j] * qq[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);

    float *state = a.state + (size_t)nh * dv * DK;
    for (int i0 = warp * kRows; i0 < dv; i0 += kWarps * kRows) {
        float s[kRows][VEC];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const V x = *reinterpret_cast<const V *>(state + (size_t)(i0 + u) * DK + lane * VEC);
            const float *xf = reinterpret_cast<const float *>(&x);
#pragma unroll
            for (int j = 0; j < VEC; ++j) s[u][j] = xf[j] * al[j];  // S~ = S Diag(alpha)
        }
        float r[kRows], o[kRows];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            r[u] = 0.f; o[u] = 0.f;
#pragma unroll
            for (int j = 0; j < VEC; ++j) { r[u] += s[u][j] * kk[j]; o[u] += s[u][j] * qq[j]; }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                r[u] += __shfl_xor_sync(0xffffffffu, r[u], off);
                o[u] += __shfl_xor_sync(0xffffffffu, o[u], off);
            }
        }
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const int i = i0 + u;
            const float vi = load_elem(a.v, (long long)nh * dv + i, a.bf16);
            const float delta = beta * (vi - r[u]);
            V y;
            float *yf = reinterpret_cast<float *>(&y);
#pragma unroll
            for (int j = 0; j < VEC; ++j) yf[j] = s[u][j] + delta * kk[j];
            *reinterpret_cast<V *>(state + (size_t)i * DK + lane * VEC) = y;
            if (lane == 0) store_elem(a.o, (long long)nh * dv + i, o[u] + delta * kq, a.bf16);
        }
    }
}

template <int DK, bool CH>
cudaError_t launch_t(const DecodeArgs &a, cudaStream_t s) {
    const long long blocks = (long long)a.N * a.H;
    if (blocks == 0) return cudaSuccess;
    decode_kernel<DK, CH><<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s, int *launches) {
    if ((long long)a.N * a.H > 0 && launches) ++*launches;
    if (a.dk == 128) return a.channel ? launch_t<128, true>(a, s) : launch_t<128, false>(a, s);
    return a.channel ? launch_t<64, true>(a, s) : launch_t<64, false>(a, s);
}

}  // namespace gdn
