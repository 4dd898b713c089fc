// gdn_chunk_tc.cu -- chunkwise gated delta rule prefill on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators, TMA-staged 128B-swizzled bf16
// tiles) for bf16 inputs with d_k = d_v = 128 and scalar (GDN) decay.
//
// One CTA (4 warps) per (sequence, head, 64-wide slice of d_v).  The fp32
// state slice lives in registers (thread c holds column c of S, i.e. row c of
// S^T) and the CTA walks the sequence's chunks of C = 64 tokens (FG2-GDN
// paper, section 3.6; the Gated Delta Networks page, section 3.3 for the scalar
// cumulative decay).  With g_r the cumulative log decay inside the chunk,
// gamma_r = e^{g_r}, every contraction is one M = 128 tcgen05.mma group:
//
//   D_kq  = [K; Q] K^T                 (A = beta_r e^{g_r-g_s} (K K^T)_rs, s < r;
//                                        P = e^{g_r-g_s} (Q K^T)_rs,      s <= r)
//   T     = (I + A)^{-1}               (blocked forward substitution, fp32, CUDA cores)
//   D_w   = (beta gamma K)^T T^T       (= W^T, W = T diag(beta)(gamma . K))
//   D_vp  = [T; 0] (beta V)            (rows 0-63: U = T diag(beta) V)
//   D_vp += [-W; gamma Q] S^T          (rows 0-63: V' = U - W S^T; rows 64-127: gamma Q S^T)
//   D_ds  = K^^T V'                    (K^_s = e^{g_C - g_s} k_s)
//   D_vp += [0; P] V'                  (rows 64-127: O = gamma Q S^T + P V')
//   S    <- e^{g_C} S + D_ds^T
//
// Operands that contract over the key channels are K-major tiles; operands that
// contract over tokens use the token-major tiles directly as MN-major
// descriptors, so no transposes go through shared memory.  This first version
// runs the phases of a chunk one after the other (the next chunk's tiles are
// prefetched by TMA while the current chunk computes).
#include <mutex>

#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr int C = kChunk;      // 64
constexpr int DK = 128;
constexpr int DVS = 64;        // d_v slice per CTA
constexpr long long kWaitLimit = 1LL << 31;  // SM cycles (~1 s) before a wait gives up

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_KQ = 0;          // [2 atom cols][128 rows: K 0-63, Q 64-127][128 B]
constexpr uint32_t OFF_VT = 32768;      // [64 rows][128 B]  V slice tile
constexpr uint32_t OFF_BK = 40960;      // beta gamma K, [2 MN blocks][64 rows][128 B]
constexpr uint32_t OFF_BV = 57344;      // beta V,       [64 rows][128 B]
constexpr uint32_t OFF_KH = 65536;      // K^,           [2 MN blocks][64 rows][128 B]
constexpr uint32_t OFF_T = 81920;       // T (bf16),     [64 rows][128 B]
constexpr uint32_t OFF_Z = 90112;       // zeros,        [64 rows][128 B]
constexpr uint32_t OFF_P = 98304;       // P (bf16),     [64 rows][128 B]
constexpr uint32_t OFF_WQ = 106496;     // [-W; gamma Q], [2 atom cols][128 rows][128 B]
constexpr uint32_t OFF_SB = 139264;     // S (bf16) MN-major: [128 rows c][64 i]
constexpr uint32_t OFF_VP = 155648;     // V' (bf16) MN-major: [64 rows r][64 i]
constexpr uint32_t OFF_AF = 163840;     // A fp32 [64][65]
constexpr uint32_t OFF_TF = OFF_AF + 64 * 65 * 4;   // T fp32 [64][65]
constexpr uint32_t OFF_XS = OFF_TF + 64 * 65 * 4;   // 3 x 16x16 fp32 scratch
constexpr uint32_t OFF_ROW = OFF_XS + 3 * 256 * 4;  // 5 x 64 fp32 per-row scalars
constexpr uint32_t OFF_BAR = OFF_ROW + 5 * 64 * 4;  // mbarriers, TMEM address, flags
constexpr uint32_t SMEM_USED = OFF_BAR + 64;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;   // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_KQ = 0, COL_W = 64, COL_VP = 128, COL_DS = 192, TMEM_COLS = 256;

constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);  // [K;Q] K^T
constexpr uint32_t ID_MK = idesc_bf16(128, 64, true, false);   // (bgK)^T T^T
constexpr uint32_t ID_KM = idesc_bf16(128, 64, false, true);   // [T;0] bV, [-W;gQ] S^T, [0;P] V'
constexpr uint32_t ID_MM = idesc_bf16(128, 64, true, true);    // K^^T V'

__device__ __forceinline__ uint4 pack8(const float *x) {
    uint4 u;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(x[0], x[1]);
    __nv_bfloat162 h1 = __floats2bfloat162_rn(x[2], x[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(x[4], x[5]);
    __nv_bfloat162 h3 = __floats2bfloat162_rn(x[6], x[7]);
    u.x = *reinterpret_cast<uint32_t *>(&h0);
    u.y = *reinterpret_cast<uint32_t *>(&h1);
    u.z = *reinterpret_cast<uint32_t *>(&h2);
    u.w = *reinterpret_cast<uint32_t *>(&h3);
    return u;
}

__device__ __forceinline__ uint4 scale8(uint4 u, float s) {
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
    float x[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        float2 f = __bfloat1622float2(h[j]);
        x[2 * j] = f.x * s;
        x[2 * j + 1] = f.y * s;
    }
    return pack8(x);
}

// Copy a 128B-swizzled tile region (rows x 8 chunks) from src to dst, scaling
// row r by scale[r].  Source and destination rows share the swizzle phase.
__device__ __forceinline__ void scaled_copy(uint8_t *sm, uint32_t src, uint32_t dst, int rows,
                                            const float *scale, int tid) {
    for (int idx = tid; idx < rows * 8; idx += kThreads) {
        const int r = idx >> 3, pj = idx & 7;
        const uint4 u = *reinterpret_cast<const uint4 *>(sm + src + r * 128 + pj * 16);
        *reinterpret_cast<uint4 *>(sm + dst + r * 128 + pj * 16) = scale8(u, scale[r]);
    }
}

__global__ void __launch_bounds__(kThreads, 1)
chunk_tc_kernel(const PrefillArgs a, const __grid_constant__ CUtensorMap tm_q,
                const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    float *AF = reinterpret_cast<float *>(sm + OFF_AF);
    float *TF = reinterpret_cast<float *>(sm + OFF_TF);
    float *XS = reinterpret_cast<float *>(sm + OFF_XS);
    float *g_s = reinterpret_cast<float *>(sm + OFF_ROW);   // cumulative log decay
    float *b_s = g_s + 64;                                  // beta
    float *bg_s = g_s + 128;                                // beta_r e^{g_r}
    float *kh_s = g_s + 192;                                // e^{g_C - g_r}
    float *gq_s = g_s + 256;                                // e^{g_r}
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 20);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nsl = a.dv / DVS;
    const int item = blockIdx.x;
    const int slice = item % nsl;
    const int h = (item / nsl) % a.H;
    const int n = item / (nsl * a.H);
    const int v0 = slice * DVS;
    const int H = a.H;

    long long t_begin, t_end;
    seq_range(a, n, &t_begin, &t_end);
    const int nchunks = (int)((t_end - t_begin + C - 1) / C);

    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int i = tid; i < 512; i += kThreads)
        reinterpret_cast<uint4 *>(sm + OFF_Z)[i] = make_uint4(0, 0, 0, 0);

    // state slice: thread c holds S[v0 + i][c] for i in [0, 64)
    float s_reg[DVS];
    const size_t st_base = ((size_t)n * H + h) * a.dv * DK;
#pragma unroll
    for (int i = 0; i < DVS; ++i)
        s_reg[i] = a.s0 ? a.s0[st_base + (size_t)(v0 + i) * DK + tid] : 0.f;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;

    // bf16 copy of the state as the MN-major B operand of [-W; gQ] S^T
    auto write_state_bf16 = [&]() {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4 *>(sm + OFF_SB + sw128(tid, j)) = pack8(s_reg + 8 * j);
    };
    write_state_bf16();

    auto issue_tma = [&](long long t0) {
        mbar_arrive_expect_tx(bar_tma, 40960);
        tma_load_3d(sm + OFF_KQ, &tm_k, 0, h, (int)t0, bar_tma);
        tma_load_3d(sm + OFF_KQ + 16384, &tm_k, 64, h, (int)t0, bar_tma);
        tma_load_3d(sm + OFF_KQ + 8192, &tm_q, 0, h, (int)t0, bar_tma);
        tma_load_3d(sm + OFF_KQ + 16384 + 8192, &tm_q, 64, h, (int)t0, bar_tma);
        tma_load_3d(sm + OFF_VT, &tm_v, v0, h, (int)t0, bar_tma);
    };

    uint32_t tma_phase = 0, mma_phase = 0;
    bool tma_pending = false, mma_pending = false;
    if (tid == 0 && nchunks > 0) {
        fence_proxy_async_smem();
        issue_tma(t_begin);
    }
    tma_pending = nchunks > 0;

    auto wait_mma = [&]() {
        if (!mbar_wait(bar_mma, mma_phase & 1, kWaitLimit)) *abort_flag = 1;
        ++mma_phase;
        mma_pending = false;
        tc_fence_after();
    };

    for (int ci = 0; ci < nchunks; ++ci) {
        const long long t0 = t_begin + (long long)ci * C;
        const int L = (t_end - t0) < C ? (int)(t_end - t0) : C;

        // ---- gates: beta and the cumulative log decay (warp 0) -----------
        if (warp == 0) {
            const int r0 = 2 * lane, r1 = 2 * lane + 1;
            const float la0 = r0 < L ? a.log_alpha[(t0 + r0) * H + h] : 0.f;
            const float la1 = r1 < L ? a.log_alpha[(t0 + r1) * H + h] : 0.f;
            const float be0 = r0 < L ? a.beta[(t0 + r0) * H + h] : 0.f;
            const float be1 = r1 < L ? a.beta[(t0 + r1) * H + h] : 0.f;
            float incl = la0 + la1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float gC = __shfl_sync(0xffffffffu, incl, 31);
            const float g1 = incl, g0 = incl - la1;
            g_s[r0] = g0; g_s[r1] = g1;
            b_s[r0] = be0; b_s[r1] = be1;
            bg_s[r0] = be0 * __expf(g0); bg_s[r1] = be1 * __expf(g1);
            kh_s[r0] = __expf(gC - g0); kh_s[r1] = __expf(gC - g1);
            gq_s[r0] = __expf(g0); gq_s[r1] = __expf(g1);
        }
        // ---- wait for this chunk's tiles ---------------------------------
        if (!mbar_wait(bar_tma, tma_phase & 1, kWaitLimit)) *abort_flag = 1;
        ++tma_phase;
        tma_pending = false;
        __syncthreads();
        if (*abort_flag) break;
        // zero the rows past the end of the sequence (they hold the next
        // sequence's tokens or TMA fill)
        if (L < C) {
            for (int idx = tid; idx < (C - L) * 8; idx += kThreads) {
                const int r = L + (idx >> 3), pj = idx & 7;
                const uint4 z = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm + OFF_KQ + r * 128 + pj * 16) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KQ + 16384 + r * 128 + pj * 16) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KQ + 8192 + r * 128 + pj * 16) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_KQ + 24576 + r * 128 + pj * 16) = z;
                *reinterpret_cast<uint4 *>(sm + OFF_VT + r * 128 + pj * 16) = z;
            }
            fence_proxy_async_smem();
            __syncthreads();
        }
        // ---- MMA 1: D_kq = [K; Q] K^T --------------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < DK / 16; ++k) {
                const uint32_t off = sbase + OFF_KQ + (k >> 2) * 16384 + (k & 3) * 32;
                const uint64_t d = desc_sw128(off, 16, 1024);
                mma_bf16(tmem + COL_KQ, d, d, ID_KK, k > 0);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        // ---- operands from the tiles (the MMA only reads them) -------------
        scaled_copy(sm, OFF_KQ, OFF_BK, 64, bg_s, tid);                 // beta gamma K, block 0
        scaled_copy(sm, OFF_KQ + 16384, OFF_BK + 8192, 64, bg_s, tid);  // block 1
        scaled_copy(sm, OFF_KQ, OFF_KH, 64, kh_s, tid);                 // K^
        scaled_copy(sm, OFF_KQ + 16384, OFF_KH + 8192, 64, kh_s, tid);
        scaled_copy(sm, OFF_KQ + 8192, OFF_WQ + 8192, 64, gq_s, tid);   // gamma Q, atom col 0
        scaled_copy(sm, OFF_KQ + 24576, OFF_WQ + 24576, 64, gq_s, tid); // atom col 1
        scaled_copy(sm, OFF_VT, OFF_BV, 64, b_s, tid);                  // beta V
        wait_mma();
        // ---- A (fp32) and P (bf16) from D_kq -------------------------------
        {
            float x[64];
            tmem_load<64>(tmem + lane_off + COL_KQ, x);
            if (warp < 2) {
                const int r = tid;
                const float gr = g_s[r], br = b_s[r];
#pragma unroll
                for (int s = 0; s < 64; ++s)
                    AF[r * 65 + s] = s < r ? br * __expf(gr - g_s[s]) * x[s] : 0.f;
            } else {
                const int r = tid - 64;
                const float gr = g_s[r];
#pragma unroll
                for (int s = 0; s < 64; ++s) x[s] = s <= r ? __expf(gr - g_s[s]) * x[s] : 0.f;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_P + sw128(r, j)) = pack8(x + 8 * j);
            }
        }
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        // the tiles are free: prefetch the next chunk while this one computes
        if (tid == 0 && ci + 1 < nchunks) {
            fence_proxy_async_smem();
            issue_tma(t0 + C);
        }
        tma_pending = ci + 1 < nchunks;
        // ---- T = (I + A)^{-1}: 16x16 diagonal blocks by forward substitution
        if (warp < 2) {
            const int blk = 2 * warp + (lane >> 4), j = lane & 15, o = 16 * blk;
            float t[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < i; ++m) acc -= AF[(o + i) * 65 + o + m] * t[m];
                t[i] = acc;
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) TF[(o + i) * 65 + o + j] = t[i];
        }
        __syncthreads();
        // off-diagonal blocks by block distance d: T_ij = -T_ii sum_{k=j}^{i-1} A_ik T_kj
        for (int d = 1; d < 4; ++d) {
            const int nb = 4 - d;
            for (int e = tid; e < nb * 256; e += kThreads) {
                const int bj = e >> 8, bi = bj + d, ii = (e >> 4) & 15, jj = e & 15;
                float acc = 0.f;
                for (int k = bj; k < bi; ++k)
#pragma unroll
                    for (int m = 0; m < 16; ++m)
                        acc += AF[(16 * bi + ii) * 65 + 16 * k + m] * TF[(16 * k + m) * 65 + 16 * bj + jj];
                XS[e] = acc;
            }
            __syncthreads();
            for (int e = tid; e < nb * 256; e += kThreads) {
                const int bj = e >> 8, bi = bj + d, ii = (e >> 4) & 15, jj = e & 15;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m)
                    acc += TF[(16 * bi + ii) * 65 + 16 * bi + m] * XS[(e & ~255) + m * 16 + jj];
                TF[(16 * bi + ii) * 65 + 16 * bj + jj] = -acc;
            }
            __syncthreads();
        }
        // T in bf16 (K-major rows r, columns s; zero above the diagonal)
        {
            const int r = tid >> 1, half = tid & 1;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int j = 4 * half + jj;
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * j + e;
                    x[e] = s <= r ? TF[r * 65 + s] : 0.f;
                }
                *reinterpret_cast<uint4 *>(sm + OFF_T + sw128(r, j)) = pack8(x);
            }
        }
        fence_proxy_async_smem();
        __syncthreads();
        // ---- MMA 2: W^T = (bgK)^T T^T;  MMA 3: D_vp = [T; 0] (bV) ---------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const uint64_t da = desc_sw128(sbase + OFF_BK + k * 2048, 8192, 1024);
                const uint64_t db = desc_sw128(sbase + OFF_T + k * 32, 16, 1024);
                mma_bf16(tmem + COL_W, da, db, ID_MK, k > 0);
            }
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const uint64_t da = desc_sw128(sbase + OFF_T + k * 32, 16, 1024);
                const uint64_t db = desc_sw128(sbase + OFF_BV + k * 2048, 8192, 1024);
                mma_bf16(tmem + COL_VP, da, db, ID_KM, k > 0);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        wait_mma();
        // ---- -W into rows 0-63 of the [-W; gamma Q] operand ----------------
        {
            float w[64];
            tmem_load<64>(tmem + lane_off + COL_W, w);  // lane c: W[r][c], r = 0..63
            const int c = tid, ac = c >> 6, cc = c & 63;
#pragma unroll
            for (int r = 0; r < 64; ++r) {
                const uint32_t off = OFF_WQ + ac * 16384 + r * 128 +
                                     ((((cc >> 3) ^ (r & 7))) << 4) + (cc & 7) * 2;
                *reinterpret_cast<__nv_bfloat16 *>(sm + off) = __float2bfloat16_rn(-w[r]);
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        // ---- MMA 4: D_vp += [-W; gamma Q] S^T ------------------------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < DK / 16; ++k) {
                const uint64_t da = desc_sw128(sbase + OFF_WQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
                const uint64_t db = desc_sw128(sbase + OFF_SB + k * 2048, 16384, 1024);
                mma_bf16(tmem + COL_VP, da, db, ID_KM, 1);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        wait_mma();
        // ---- V' (rows 0-63 of D_vp) as the MN-major operand ---------------
        if (warp < 2) {
            float vp[64];
            tmem_load<64>(tmem + lane_off + COL_VP, vp);
            const int r = tid;
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sm + OFF_VP + sw128(r, j)) = pack8(vp + 8 * j);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (*abort_flag) break;
        // ---- MMA 5: D_ds = K^^T V';  MMA 6: D_vp += [0; P] V' --------------
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const uint64_t da = desc_sw128(sbase + OFF_KH + k * 2048, 8192, 1024);
                const uint64_t db = desc_sw128(sbase + OFF_VP + k * 2048, 8192, 1024);
                mma_bf16(tmem + COL_DS, da, db, ID_MM, k > 0);
            }
#pragma unroll
            for (int k = 0; k < C / 16; ++k) {
                const uint64_t da = desc_sw128(sbase + OFF_Z + k * 32, 16, 1024);
                const uint64_t db = desc_sw128(sbase + OFF_VP + k * 2048, 8192, 1024);
                mma_bf16(tmem + COL_VP, da, db, ID_KM, 1);
            }
            mma_commit(bar_mma);
        }
        mma_pending = true;
        wait_mma();
        // ---- state update and output ---------------------------------------
        {
            float ds[64];
            tmem_load<64>(tmem + lane_off + COL_DS, ds);  // lane c: dS[i][c]
            const float dec = __expf(g_s[63]);
#pragma unroll
            for (int i = 0; i < DVS; ++i) s_reg[i] = dec * s_reg[i] + ds[i];
        }
        if (warp >= 2) {
            float o[64];
            tmem_load<64>(tmem + lane_off + COL_VP, o);
            const int r = tid - 64;
            if (r < L) {
                __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.o) +
                                     ((t0 + r) * H + h) * (long long)a.dv + v0;
#pragma unroll
                for (int j = 0; j < 8; ++j) reinterpret_cast<uint4 *>(dst)[j] = pack8(o + 8 * j);
            }
        }
        write_state_bf16();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
    }

    // ---- final state, cleanup -------------------------------------------------
    if (*abort_flag) {
        if (tid == 0) atomicOr(a.err, kErrTimeout);
        // let copies and MMAs already issued land before the CTA exits
        if (tma_pending) mbar_wait(bar_tma, tma_phase & 1, kWaitLimit);
        if (mma_pending) mbar_wait(bar_mma, mma_phase & 1, kWaitLimit);
    } else if (a.s_final) {
#pragma unroll
        for (int i = 0; i < DVS; ++i) a.s_final[st_base + (size_t)(v0 + i) * DK + tid] = s_reg[i];
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// ------------------------------------------------------------------- host --
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// [tokens, H, d] bf16 viewed as a 3-D tensor (d, H, tokens); box 64 x 1 x 64.
bool make_map(CUtensorMap *m, const void *base, int d, int H, long long ntok) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)ntok};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

}  // namespace

bool chunk_tc_supported(const gdn_dims &d) {
    return d.dtype == GDN_BF16 && d.d_k == DK && d.d_v == 128 && d.decay == GDN_DECAY_SCALAR &&
           (long long)d.B * d.T < (1LL << 31);
}

size_t chunk_tc_scratch_bytes(const gdn_dims &) { return 0; }

cudaError_t launch_chunk_tc(const PrefillArgs &a, cudaStream_t s, int *launches) {
    const long long items = (long long)a.n_seqs * a.H * (a.dv / DVS);
    const long long ntok = (long long)a.B * a.T;
    if (items == 0) return cudaSuccess;
    if (ntok == 0) {
        // no tokens at all: every sequence is empty, final = initial state
        if (a.s_final && a.s_final != a.s0) {
            const size_t bytes = (size_t)a.n_seqs * a.H * a.dv * a.dk * sizeof(float);
            return a.s0 ? cudaMemcpyAsync(a.s_final, a.s0, bytes, cudaMemcpyDeviceToDevice, s)
                        : cudaMemsetAsync(a.s_final, 0, bytes, s);
        }
        return cudaSuccess;
    }
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, a.q, a.dk, a.H, ntok) || !make_map(&mk, a.k, a.dk, a.H, ntok) ||
        !make_map(&mv, a.v, a.dv, a.H, ntok))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    chunk_tc_kernel<<<(unsigned)items, kThreads, SMEM_BYTES, s>>>(a, mq, mk, mv);
    if (launches) ++*launches;
    return cudaGetLastError();
}

}  // namespace gdn
