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
// consecutive columns; kRows (8) rows are in flight per warp and stay in registers
// across the K tokens, so the state is read once and written at most once.
#include "gdn_internal.cuh"

namespace gdn {
namespace {

constexpr int kWarps = 4;
constexpr int kRows = 8;

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

// One token of the recurrence on kRows state rows of this warp (rows i0 ..),
// lane's columns; writes the outputs of the rows when `out`.  The 2 kRows row
// sums (r_u = S~_u . k, o_u = S~_u . q) are reduced across the warp by a
// transposed butterfly: at each of the first four levels a lane keeps half of its
// values and adds its partner's copy of them, so 16 values take 8 + 4 + 2 + 1 + 1
// shuffles and lane l ends with value 8 b4 + 4 b3 + 2 b2 + b1 (l's bits): r_u in
// lanes 2u, 2u + 1 and o_u in lanes 16 + 2u, 16 + 2u + 1.  Each r_u then goes to
// every lane for the update, and lane 16 + 2u writes row u's output.
template <int DK, bool CH>
__device__ __forceinline__ void token_step(const VerifyArgs &a, long long tok, int i0, int lane,
                                           float (&s)[kRows][DK / 32], bool out) {
    static_assert(kRows == 8, "the butterfly below reduces 2 x 8 values");
    constexpr int VEC = DK / 32;
    const int dv = a.dv;
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
    float p[16];  // r_0 .. r_7, o_0 .. o_7 (this lane's columns)
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
        p[u] = 0.f; p[8 + u] = 0.f;
#pragma unroll
        for (int j = 0; j < VEC; ++j) {
            s[u][j] *= al[j];  // S~ = S Diag(alpha)
            p[u] += s[u][j] * kk[j];
            p[8 + u] += s[u][j] * qq[j];
        }
    }
    float p8[8], p4[4], p2[2];
    const bool b4 = lane & 16, b3 = lane & 8, b2 = lane & 4, b1 = lane & 2;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float keep = b4 ? p[8 + j] : p[j], give = b4 ? p[j] : p[8 + j];
        p8[j] = keep + __shfl_xor_sync(0xffffffffu, give, 16);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float keep = b3 ? p8[4 + j] : p8[j], give = b3 ? p8[j] : p8[4 + j];
        p4[j] = keep + __shfl_xor_sync(0xffffffffu, give, 8);
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float keep = b2 ? p4[2 + j] : p4[j], give = b2 ? p4[j] : p4[2 + j];
        p2[j] = keep + __shfl_xor_sync(0xffffffffu, give, 4);
    }
    float v1;
    {
        const float keep = b1 ? p2[1] : p2[0], give = b1 ? p2[0] : p2[1];
        v1 = keep + __shfl_xor_sync(0xffffffffu, give, 2);
    }
    v1 += __shfl_xor_sync(0xffffffffu, v1, 1);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    // this lane's output row (lanes 16 + 2u) and its r
    const int uo = (lane >> 1) & 7;
    const float r_o = __shfl_sync(0xffffffffu, v1, 2 * uo);
#pragma unroll
    for (int u = 0; u < kRows; ++u) {
        const float r = __shfl_sync(0xffffffffu, v1, 2 * u);
        const float vi = load_elem(a.v, tok * dv + i0 + u, a.bf16);
        const float delta = beta * (vi - r);
#pragma unroll
        for (int j = 0; j < VEC; ++j) s[u][j] += delta * kk[j];
    }
    if (out && lane >= 16 && !(lane & 1)) {
        const int i = i0 + uo;
        const float delta = beta * (load_elem(a.v, tok * dv + i, a.bf16) - r_o);
        store_elem(a.o, tok * dv + i, v1 + delta * kq, a.bf16);
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
            token_step<DK, CH>(a, tok, i0, lane, s, a.o != nullptr);
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

// Tree-shaped drafts: node j's token follows its parent's (parent[n][j] in
// [-1, j - 1]; -1: the current state; anything else is taken as -1).  Node j's
// output is S_j q_j, S_j the state after the path from the current state to j;
// n_commit[n] = c >= 1 commits the state after node c - 1's path.  Each node's
// root-first path is tabulated in shared memory; a warp walks a node's path from
// the current state of its rows (read from the state buffer), except that a node
// whose parent is the node just done continues from that state (a chain of
// drafts costs one step per node).
constexpr int kMaxTree = kMaxTreeNodes;

template <int DK, bool CH>
__global__ void __launch_bounds__(kWarps * 32)
verify_tree_kernel(VerifyArgs a) {
    constexpr int VEC = DK / 32;
    using V = typename VecF<VEC>::T;
    __shared__ int anc[kMaxTree][kMaxTree];
    __shared__ int depth[kMaxTree];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nh = blockIdx.x;  // n * H + h
    const int n = nh / a.H, h = nh % a.H;
    const int dv = a.dv, K = a.K;
    const int commit = a.n_commit ? min(max(a.n_commit[n], 0), K) : 0;
    if (!a.o && commit == 0) return;
    const int32_t *par = a.parent + (size_t)n * K;
    auto parent_of = [&](int x) {
        const int p = par[x];
        return (p >= 0 && p < x) ? p : -1;
    };
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
        int d = 0;
        for (int x = j; x >= 0; x = parent_of(x)) ++d;
        depth[j] = d;
        int i = d - 1;
        for (int x = j; x >= 0; x = parent_of(x)) anc[j][i--] = x;
    }
    __syncthreads();

    float *state = a.state + (size_t)nh * dv * DK;
    auto tok_of = [&](int x) { return ((long long)n * K + x) * a.H + h; };
    for (int i0 = warp * kRows; i0 < dv; i0 += kWarps * kRows) {
        float s[kRows][VEC];
        // s holds the state after node `cur`'s path (-2: nothing yet).  Targets: the
        // K nodes when the outputs are wanted, then the committed node.
        int cur = -2;
        for (int it = 0; it <= K; ++it) {
            int x;
            bool out_last;
            if (it < K) {
                if (!a.o) continue;
                x = it;
                out_last = true;
            } else {
                if (commit == 0) break;
                x = commit - 1;
                out_last = false;
            }
            if (x != cur) {
                const int d = depth[x];
                const int px = d >= 2 ? anc[x][d - 2] : -1;
                int i = d - 1;  // continue from cur when it is x's parent
                if (px != cur) {
                    // restart from the current state of these rows (the state
                    // buffer: the commit below writes it only after its last read)
#pragma unroll
                    for (int u = 0; u < kRows; ++u) {
                        const V y = *reinterpret_cast<const V *>(state + (size_t)(i0 + u) * DK + lane * VEC);
                        const float *yf = reinterpret_cast<const float *>(&y);
#pragma unroll
                        for (int j = 0; j < VEC; ++j) s[u][j] = yf[j];
                    }
                    i = 0;
                }
                for (; i < d; ++i) {
                    const int t = anc[x][i];
                    token_step<DK, CH>(a, ((long long)n * K + t) * a.H + h, i0, lane, s,
                                       out_last && i == d - 1);
                }
                cur = x;
            }
            if (it == K) {
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
    if (a.parent)
        verify_tree_kernel<DK, CH><<<(unsigned)blocks, kWarps * 32, 0, s>>>(a);
    else
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
