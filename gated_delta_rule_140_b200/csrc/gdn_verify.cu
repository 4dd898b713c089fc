// gdn_verify.cu -- multi-token verification for speculative decoding: K draft
// tokens per sequence run through the recurrence from the current state, with
// the outputs of all K and a commit of the state after the first n_commit[n].
//
// The recurrence is the decode step's (FG2-GDN section 1; o_t = S_t q_t), token
// after token.  For every (sequence, head) and state row i:
//   GDN:  r = S_i.k_t, s = S_i.q_t, delta = beta_t (v_ti - alpha_t r),
//         o_ti = alpha_t s + delta (k_t.q_t),   S_i <- alpha_t S_i + delta k_t
//   KDA:  S~_i = S_i . alpha_t, r = S~_i.k_t, s = S~_i.q_t, delta = beta_t (v_ti - r),
//         o_ti = s + delta (k_t.q_t),   S_i <- S~_i + delta k_t
// A draft is peeked (outputs, state untouched) and then committed up to the
// accepted length, so no per-position state is ever stored: the state after
// j tokens is recomputed from the state before them and the j tokens (the
// speculative-decoding use the Gated DeltaNet-2 page's TreeWY finding describes,
// for a chain of drafts).
//
// Layout as the decode step's: a warp owns whole state rows, each lane DK/32
// consecutive columns; kRows rows are in flight per warp and stay in registers
// across the K tokens, so the state is read once and written at most once.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kWarps = 4;
constexpr int kRows = 4;

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
verify_kernel(VerifyArgs a) {
    constexpr int VEC = DK / 32;
    using V = typename VecF<VEC>::T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nh = blockIdx.x;  // n * H + h
    const int n = nh / a.H, h = nh % a.H;
    const int dv = a.dv, K = a.K;
    // the state after `commit` tokens is written back (0: untouched)
    const int commit = a.n_commit ? min(max(a.n_commit[n], 0), K) : 0;
    // tokens to run: all K when the outputs are wanted, else only the committed ones
    const int steps = a.o ? K : commit;
    if (steps == 0) return;

    float *state = a.state + (size_t)nh * dv * DK;
    for (int i0 = warp * kRows; i0 < dv; i0 += kWarps * kRows) {
        float s[kRows][VEC];
#pragma unroll
        for (int u = 0; u < kRows; ++u) {
            const V x = *reinterpret_cast<const V *>(state + (size_t)(i0 + u) * DK + lane * VEC);
            const float *xf = reinterpret_cast<const float *>(&x);
#pragma unroll
            for (int j = 0; j < VEC; ++j) s[u][j] = xf[j];
        }
        for (int t = 0; t < steps; ++t) {
            const long long tok = ((long long)n * K + t) * a.H + h;  // token-major [N, K, H]
            float kk[VEC], qq[VEC], al[VEC];
            load_vec(a.k, tok * DK + lane * VEC, a.bf16, kk, VEC);
            load_vec(a.q, tok * DK + lane * VEC, a.bf16, qq, VEC);
            const float beta = a.beta[tok];
            if (CH) {
#pragma unroll
                for (int j = 0; j < VEC; ++j) al[j] = expf(a.log_alpha[tok * DK + lane * VEC + j]);
            } else {
                const float alpha = expf(a.log_alpha[tok]);
#pragma unroll
                for (int j = 0; j < VEC; ++j) al[j] = alpha;
            }
            float kq = 0.f;
#pragma unroll
            for (int j = 0; j < VEC; ++j) kq += kk[j] * qq[j];
            float r[kRows], o[kRows];
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                r[u] = 0.f; o[u] = 0.f;
#pragma unroll
                for (int j = 0; j < VEC; ++j) {
                    s[u][j] *= al[j];  // S~ = S Diag(alpha)
                    r[u] += s[u][j] * kk[j];
                    o[u] += s[u][j] * qq[j];
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
                for (int u = 0; u < kRows; ++u) {
                    r[u] += __shfl_xor_sync(0xffffffffu, r[u], off);
                    o[u] += __shfl_xor_sync(0xffffffffu, o[u], off);
                }
            }
#pragma unroll
            for (int u = 0; u < kRows; ++u) {
                const int i = i0 + u;
                const float vi = load_elem(a.v, tok * dv + i, a.bf16);
                const float delta = beta * (vi - r[u]);
#pragma unroll
                for (int j = 0; j < VEC; ++j) s[u][j] += delta * kk[j];
                if (a.o && lane == 0) store_elem(a.o, tok * dv + i, o[u] + delta * kq, a.bf16);
            }
            if (t + 1 == commit) {
#pragma unroll
                for (int u = 0; u < kRows; ++u) {
                    V y;
                    float *yf = reinterpret_cast<float *>(&y);
#pragma unroll
                    for (int j = 0; j < VEC; ++j) yf[j] = s[u][j];
                    *reinterpret_cast<V *>(state + (size_t)(i0 + u) * DK + lane * VEC) = y;
                }
            }
        }
    }
}

template <int DK, bool CH>
cudaError_t launch_t(const VerifyArgs &a, cudaStream_t s) {
    const long long blocks = (long long)a.N * a.H;
    if (blocks == 0 || a.K == 0) return cudaSuccess;
    verify_kernel<DK, CH><<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_verify(const VerifyArgs &a, cudaStream_t s, int *launches) {
    if ((long long)a.N * a.H > 0 && a.K > 0 && launches) ++*launches;
    if (a.dk == 128) return a.channel ? launch_t<128, true>(a, s) : launch_t<128, false>(a, s);
    return a.channel ? launch_t<64, true>(a, s) : launch_t<64, false>(a, s);
}

}  // namespace gdn
