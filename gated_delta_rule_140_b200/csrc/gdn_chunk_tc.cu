// gdn_chunk_tc.cu -- chunkwise gated delta rule prefill on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators, TMA-staged 128B-swizzled bf16
// tiles) for bf16 inputs with d_k = d_v = 128 and scalar (GDN) decay.
//
// One CTA per (sequence, head, 64-wide slice of d_v), walking the sequence's
// chunks of C = 64 tokens (FG2-GDN paper, section 3.6: WY representation and
// UT transform inside a chunk, inter-chunk state propagation, intra-chunk
// causal product; the Gated Delta Networks page, section 3.3, for the scalar
// cumulative decay g_r, gamma_r = e^{g_r}).  Per chunk:
//
//   D_kq  = [Q; K] K^T                  rows 0-63: Q K^T, rows 64-127: K K^T
//   A_rs  = beta_r e^{g_r-g_s} (K K^T)_rs, s < r;  P_rs = e^{g_r-g_s} (Q K^T)_rs, s <= r
//   T     = (I + A)^{-1}                 blocked forward substitution, fp32
//   T_b   = T diag(beta),  T_bg = T diag(beta gamma)       (bf16)
//   D_w   = K^T T_bg^T                   = W^T,  W = T diag(beta)(gamma . K)
//   D_vp  = [T_b; 0] V                   rows 0-63: U = T diag(beta) V
//   D_vp += [-W; gamma Q] S^T            rows 0-63: V' = U - W S^T; rows 64-127: gamma Q S^T
//   D_ds  = K^^T V',  K^_s = e^{g_C-g_s} k_s
//   D_vp += [0; P] V'                    rows 64-127: O = gamma Q S^T + P V'
//   S    <- e^{g_C} S + D_ds^T
//
// Warp roles (384 threads):
//   warps 0-7  "local": everything that depends only on the chunk's own tokens
//              (the first four and the "W/U" MMAs, A, T, W, P, K^, gamma Q),
//              one chunk ahead of the state warps;
//   warps 8-11 "state": the sequential inter-chunk pass (the [-W; gamma Q] S^T,
//              K^^T V' and [0; P] V' MMAs, the fp32 state in registers --
//              thread c holds column c of the state slice -- and the output).
// The groups hand chunks over through mbarriers; tiles arrive by TMA into a
// two-stage ring.  Every wait is bounded: on expiry the kernel records
// kErrTimeout, both groups leave their loops at the next barrier, in-flight
// copies and MMAs are drained (again with a bound) and TMEM is freed.
#include "gdn_internal.cuh"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int C = kChunk;       // 64
constexpr int DK = 128;
constexpr int DVS = 64;         // d_v slice per CTA
constexpr int kLocal = 256;     // threads of the local group
constexpr int kState = 128;     // threads of the state group
constexpr int kThreads = kLocal + kState;
constexpr int BAR_LOCAL = 1, BAR_STATE = 2;  // named barrier ids
constexpr long long kWaitLimit = 1LL << 31;   // SM cycles (~1 s)
constexpr int LDA = 68;         // fp32 row stride of A and T in smem

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_RAW = 0;          // 2 stages x 40 KB: [Q|K atom col 0][Q|K atom col 1][V]
constexpr uint32_t RAW_STAGE = 40960;
constexpr uint32_t RAW_K = 8192;         //   K rows follow Q rows inside an atom column
constexpr uint32_t RAW_AC = 16384;       //   atom column stride
constexpr uint32_t RAW_V = 32768;
constexpr uint32_t OFF_WQ = 81920;       // [-W; gamma Q]: [atom col][128 rows][128 B]
constexpr uint32_t OFF_KH = 114688;      // K^: 2 MN blocks x [64 rows][128 B]
constexpr uint32_t OFF_TB = 131072;      // T diag(beta)  [64 rows][128 B]
constexpr uint32_t OFF_Z = 139264;       // zeros         [64 rows][128 B]
constexpr uint32_t OFF_P = 147456;       // P             [64 rows][128 B]
constexpr uint32_t OFF_TG = 155648;      // T diag(beta gamma)
constexpr uint32_t OFF_VP = 163840;      // V' MN-major   [64 rows r][64 i]
constexpr uint32_t OFF_SB = 172032;      // S bf16 MN-major [128 rows c][64 i]
constexpr uint32_t OFF_AF = 188416;      // A fp32 [64][LDA]
constexpr uint32_t OFF_TF = OFF_AF + 64 * LDA * 4;   // T fp32 [64][LDA]
constexpr uint32_t OFF_ROW = OFF_TF + 64 * LDA * 4;  // per-row scalars, 5 x 64 fp32
constexpr uint32_t OFF_HAND = OFF_ROW + 5 * 64 * 4;  // g_C of the two chunks in flight
constexpr uint32_t OFF_BAR = OFF_HAND + 64;
constexpr uint32_t SMEM_USED = OFF_BAR + 128;
constexpr uint32_t SMEM_BYTES = SMEM_USED + 1024;    // + alignment slack

// TMEM columns (fp32 accumulators, 128 lanes each)
constexpr uint32_t COL_KQ = 0;    // 2 buffers x 64
constexpr uint32_t COL_W = 128;
constexpr uint32_t COL_VP = 192;  // 2 buffers x 64
constexpr uint32_t COL_DS = 320;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_KK = idesc_bf16(128, 64, false, false);  // [Q;K] K^T
constexpr uint32_t ID_MK = idesc_bf16(128, 64, true, false);   // K^T T_bg^T
constexpr uint32_t ID_KM = idesc_bf16(128, 64, false, true);   // [T_b;0] V, [-W;gQ] S^T, [0;P] V'
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

// Wait with a bound; gives up early when the other group has aborted.
__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, volatile int *abort) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (*abort) return false;
        if (clock64() - t0 > kWaitLimit) {
            *abort = 1;
            return false;
        }
    }
    return true;
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
    float *g_s = reinterpret_cast<float *>(sm + OFF_ROW);  // cumulative log decay g_r
    float *b_s = g_s + 64;                                 // beta_r
    float *bg_s = g_s + 128;                               // beta_r e^{g_r}
    float *kh_s = g_s + 192;                               // e^{g_C - g_r}
    float *gq_s = g_s + 256;                               // e^{g_r}
    float *hand_gc = reinterpret_cast<float *>(sm + OFF_HAND);  // e^{g_C}, by chunk parity
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + OFF_BAR);
    uint64_t *bar_tma = bars + 0;     // [2] tiles of a stage landed
    uint64_t *bar_l = bars + 2;       // local MMAs done
    uint64_t *bar_s = bars + 3;       // state MMAs done
    uint64_t *bar_wqfree = bars + 4;  // [-W; gamma Q] consumed by the state MMA
    uint64_t *bar_pfree = bars + 5;   // P and K^ consumed by the state MMAs
    uint64_t *bar_vpfree = bars + 6;  // [2] output accumulator of a stage read out
    uint64_t *bar_ready = bars + 8;   // a chunk's operands are ready for the state pass
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + OFF_BAR + 80);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + OFF_BAR + 84);

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
    const size_t st_base = ((size_t)n * H + h) * a.dv * DK;

    if (warp == 0) tmem_alloc(tmem_slot, TMEM_COLS);
    if (tid == 0) {
        for (int i = 0; i < 9; ++i) mbar_init(bars + i, 1);
        fence_mbar_init();
        *abort_flag = 0;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
    }
    for (int i = tid; i < 512; i += kThreads)
        reinterpret_cast<uint4 *>(sm + OFF_Z)[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();

    // the state group's registers: thread c holds S[v0 + i][c], i in [0, 64)
    float s_reg[DVS];
    const int c_st = tid - kLocal;  // state thread index = key channel
    if (tid >= kLocal) {
#pragma unroll
        for (int i = 0; i < DVS; ++i)
            s_reg[i] = a.s0 ? a.s0[st_base + (size_t)(v0 + i) * DK + c_st] : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j)
            *reinterpret_cast<uint4 *>(sm + OFF_SB + sw128(c_st, j)) = pack8(s_reg + 8 * j);
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    auto chunk_len = [&](int m) -> int {
        const long long rem = t_end - (t_begin + (long long)m * C);
        return rem < C ? (int)rem : C;
    };

    if (tid < kLocal) {
        // ============================ local group ============================
        const int lq = warp & 3, lhalf = warp >> 2;  // TMEM lane quadrant, column half
        const uint32_t lane_off = (uint32_t)(32 * lq) << 16;
        uint32_t bl_wait = 0, bl_commit = 0;  // completions waited on / committed to bar_l
        int tma_issued[2] = {0, 0}, tma_seen[2] = {0, 0};

        auto issue_tma = [&](int m) {  // leader only
            const int st = m & 1;
            const long long t0 = t_begin + (long long)m * C;
            uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(&bar_tma[st], RAW_STAGE);
            tma_load_3d(raw, &tm_q, 0, h, (int)t0, &bar_tma[st]);
            tma_load_3d(raw + RAW_AC, &tm_q, 64, h, (int)t0, &bar_tma[st]);
            tma_load_3d(raw + RAW_K, &tm_k, 0, h, (int)t0, &bar_tma[st]);
            tma_load_3d(raw + RAW_AC + RAW_K, &tm_k, 64, h, (int)t0, &bar_tma[st]);
            tma_load_3d(raw + RAW_V, &tm_v, v0, h, (int)t0, &bar_tma[st]);
        };
        // wait for chunk m's tiles, zero rows past the sequence end, issue D_kq
        auto start_chunk = [&](int m) -> bool {
            const int st = m & 1;
            bool ok = wait_bar(&bar_tma[st], (uint32_t)(tma_seen[st] & 1), abort_flag);
            ++tma_seen[st];
            const int L = chunk_len(m);
            if (L < C) {
                uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
                for (int idx = tid; idx < (C - L) * 8; idx += kLocal) {
                    const int r = L + (idx >> 3), pj = idx & 7;
                    const uint4 z = make_uint4(0, 0, 0, 0);
                    const uint32_t o = r * 128 + pj * 16;
                    *reinterpret_cast<uint4 *>(raw + o) = z;                   // Q ac0
                    *reinterpret_cast<uint4 *>(raw + RAW_AC + o) = z;          // Q ac1
                    *reinterpret_cast<uint4 *>(raw + RAW_K + o) = z;           // K ac0
                    *reinterpret_cast<uint4 *>(raw + RAW_AC + RAW_K + o) = z;  // K ac1
                    *reinterpret_cast<uint4 *>(raw + RAW_V + o) = z;           // V
                }
                fence_proxy_async_smem();
            }
            const bool ab = named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag);
            if (ab) return false;
            if (tid == 0) {
                tc_fence_after();
                const uint32_t raw = sbase + OFF_RAW + st * RAW_STAGE;
#pragma unroll
                for (int k = 0; k < DK / 16; ++k) {
                    const uint32_t off = (k >> 2) * RAW_AC + (k & 3) * 32;
                    mma_bf16(tmem + COL_KQ + 64 * st, desc_sw128(raw + off, 16, 1024),
                             desc_sw128(raw + RAW_K + off, 16, 1024), ID_KK, k > 0);
                }
                mma_commit(bar_l);
            }
            ++bl_commit;
            return true;
        };

        if (tid == 0) {
            if (nchunks > 0) { issue_tma(0); ++tma_issued[0]; }
            if (nchunks > 1) { issue_tma(1); ++tma_issued[1]; }
        } else {
            if (nchunks > 0) ++tma_issued[0];
            if (nchunks > 1) ++tma_issued[1];
        }
        bool alive = nchunks > 0 ? start_chunk(0) : true;

        for (int m = 0; alive && m < nchunks; ++m) {
            const int st = m & 1;
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m);
            uint8_t *raw = sm + OFF_RAW + st * RAW_STAGE;
            const uint32_t raw_a = sbase + OFF_RAW + st * RAW_STAGE;
            bool ok = true;

            // ---- gates: beta and the cumulative log decay (warp 0) ------------
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
                if (lane == 0) hand_gc[st] = __expf(gC);
            }
            // ---- D_kq of this chunk ----------------------------------------------
            ok &= wait_bar(bar_l, bl_wait & 1, abort_flag);
            ++bl_wait;
            tc_fence_after();
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            // A rows (K K^T: TMEM lanes 64-127), this thread's half of the columns
            if (lq >= 2) {
                float x[32];
                tmem_load<32>(tmem + lane_off + COL_KQ + 64 * st + 32 * lhalf, x);
                const int r = 32 * (lq - 2) + lane;
                const float gr = g_s[r], br = b_s[r];
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    float4 y;
                    const int s = 32 * lhalf + j;
                    y.x = s + 0 < r ? br * __expf(gr - g_s[s + 0]) * x[j + 0] : 0.f;
                    y.y = s + 1 < r ? br * __expf(gr - g_s[s + 1]) * x[j + 1] : 0.f;
                    y.z = s + 2 < r ? br * __expf(gr - g_s[s + 2]) * x[j + 2] : 0.f;
                    y.w = s + 3 < r ? br * __expf(gr - g_s[s + 3]) * x[j + 3] : 0.f;
                    *reinterpret_cast<float4 *>(AF + r * LDA + s) = y;
                }
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- T = (I + A)^{-1} ------------------------------------------------
            // 16x16 diagonal blocks: warp w < 4 inverts block w, lane j < 16
            // owns column j (forward substitution down the column).
            if (warp < 4 && lane < 16) {
                const int o = 16 * warp, j = lane;
                float t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    float acc = (i == j) ? 1.f : 0.f;
#pragma unroll
                    for (int mm = 0; mm < i; ++mm) acc -= AF[(o + i) * LDA + o + mm] * t[mm];
                    t[i] = acc;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) TF[(o + i) * LDA + o + j] = t[i];
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // 32x32 halves: T_10 = -T_11 (A_10 T_00), T_32 = -T_33 (A_32 T_22).
            // X goes to the unused upper-right 16x16 block of each half.
            {
                const int hf = tid >> 7, e = tid & 127, ii = e >> 3, jj = 2 * (e & 7);
                const int o = 32 * hf;  // half origin
                float x0 = 0.f, x1 = 0.f;
#pragma unroll
                for (int mm = 0; mm < 16; ++mm) {
                    const float av = AF[(o + 16 + ii) * LDA + o + mm];
                    x0 += av * TF[(o + mm) * LDA + o + jj];
                    x1 += av * TF[(o + mm) * LDA + o + jj + 1];
                }
                TF[(o + ii) * LDA + o + 16 + jj] = x0;
                TF[(o + ii) * LDA + o + 16 + jj + 1] = x1;
                named_bar_sync(BAR_LOCAL, kLocal);
                float y0 = 0.f, y1 = 0.f;
#pragma unroll
                for (int mm = 0; mm < 16; ++mm) {
                    const float tv = TF[(o + 16 + ii) * LDA + o + 16 + mm];
                    y0 += tv * TF[(o + mm) * LDA + o + 16 + jj];
                    y1 += tv * TF[(o + mm) * LDA + o + 16 + jj + 1];
                }
                TF[(o + 16 + ii) * LDA + o + jj] = -y0;
                TF[(o + 16 + ii) * LDA + o + jj + 1] = -y1;
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // full: T_{H1,H0} = -T_{H1} (A_{H1,H0} T_{H0}); X in the upper-right
            // 32x32 block.  Thread: row i, four columns j4..j4+3.
            {
                const int i = tid >> 3, j4 = 4 * (tid & 7);
                float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = 0; k < 32; ++k) {
                    const float av = AF[(32 + i) * LDA + k];
                    const float4 tv = *reinterpret_cast<const float4 *>(TF + k * LDA + j4);
                    // T_{H0} is lower triangular: entries with k < j are zero, but
                    // the upper part of TF holds scratch, so mask by column.
                    x.x += (k >= j4 + 0) ? av * tv.x : 0.f;
                    x.y += (k >= j4 + 1) ? av * tv.y : 0.f;
                    x.z += (k >= j4 + 2) ? av * tv.z : 0.f;
                    x.w += (k >= j4 + 3) ? av * tv.w : 0.f;
                }
                *reinterpret_cast<float4 *>(TF + i * LDA + 32 + j4) = x;
                named_bar_sync(BAR_LOCAL, kLocal);
                float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int k = 0; k <= i; ++k) {
                    const float tv = TF[(32 + i) * LDA + 32 + k];
                    const float4 xv = *reinterpret_cast<const float4 *>(TF + k * LDA + 32 + j4);
                    y.x += tv * xv.x; y.y += tv * xv.y; y.z += tv * xv.z; y.w += tv * xv.w;
                }
                *reinterpret_cast<float4 *>(TF + (32 + i) * LDA + j4) =
                    make_float4(-y.x, -y.y, -y.z, -y.w);
            }
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- T diag(beta) and T diag(beta gamma) in bf16 (K-major, s cols) ---
            for (int idx = tid; idx < 64 * 8; idx += kLocal) {
                const int r = idx >> 3, j = idx & 7;
                float tb[8], tg[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int s = 8 * j + e;
                    const float tv = s < r ? TF[r * LDA + s] : (s == r ? 1.f : 0.f);
                    tb[e] = tv * b_s[s];
                    tg[e] = tv * bg_s[s];
                }
                *reinterpret_cast<uint4 *>(sm + OFF_TB + sw128(r, j)) = pack8(tb);
                *reinterpret_cast<uint4 *>(sm + OFF_TG + sw128(r, j)) = pack8(tg);
            }
            fence_proxy_async_smem();
            named_bar_sync(BAR_LOCAL, kLocal);
            // ---- W^T = K^T T_bg^T;  D_vp = [T_b; 0] V ------------------------------
            if (tid == 0) {
                if (m >= 2) ok &= wait_bar(&bar_vpfree[st], (uint32_t)(((m >> 1) - 1) & 1), abort_flag);
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_W, desc_sw128(raw_a + RAW_K + k * 2048, RAW_AC, 1024),
                             desc_sw128(sbase + OFF_TG + k * 32, 16, 1024), ID_MK, k > 0);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_VP + 64 * st, desc_sw128(sbase + OFF_TB + k * 32, 16, 1024),
                             desc_sw128(raw_a + RAW_V + k * 2048, 8192, 1024), ID_KM, k > 0);
                mma_commit(bar_l);
            }
            ++bl_commit;
            // ---- while those run: P, K^ and gamma Q (once the state group has
            // consumed the previous chunk's copies) --------------------------------
            if (m >= 1) {
                ok &= wait_bar(bar_pfree, (uint32_t)((m - 1) & 1), abort_flag);
                ok &= wait_bar(bar_wqfree, (uint32_t)((m - 1) & 1), abort_flag);
            }
            if (lq < 2) {  // P rows from Q K^T (TMEM lanes 0-63)
                float x[32];
                tmem_load<32>(tmem + lane_off + COL_KQ + 64 * st + 32 * lhalf, x);
                const int r = 32 * lq + lane;
                const float gr = g_s[r];
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int s = 32 * lhalf + j;
                    x[j] = s <= r ? __expf(gr - g_s[s]) * x[j] : 0.f;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_P + sw128(r, 4 * lhalf + j)) = pack8(x + 8 * j);
            }
            for (int idx = tid; idx < 1024; idx += kLocal) {
                const int b = idx >> 9, rem = idx & 511, r = rem >> 3, pj = rem & 7;
                const uint32_t o = r * 128 + pj * 16;
                const uint4 kv = *reinterpret_cast<const uint4 *>(raw + b * RAW_AC + RAW_K + o);
                *reinterpret_cast<uint4 *>(sm + OFF_KH + b * 8192 + o) = scale8(kv, kh_s[r]);
                const uint4 qv = *reinterpret_cast<const uint4 *>(raw + b * RAW_AC + o);
                *reinterpret_cast<uint4 *>(sm + OFF_WQ + b * 16384 + 8192 + o) = scale8(qv, gq_s[r]);
            }
            // ---- -W into rows 0-63 of [-W; gamma Q] --------------------------------
            ok &= wait_bar(bar_l, bl_wait & 1, abort_flag);
            ++bl_wait;
            tc_fence_after();
            {
                float w[32];
                tmem_load<32>(tmem + lane_off + COL_W + 32 * lhalf, w);  // lane c: W[r][c]
                const int c = 32 * lq + lane, ac = c >> 6, cc = c & 63;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int r = 32 * lhalf + j;
                    const uint32_t off = OFF_WQ + ac * 16384 + r * 128 +
                                         (((cc >> 3) ^ (r & 7)) << 4) + (cc & 7) * 2;
                    *reinterpret_cast<__nv_bfloat16 *>(sm + off) = __float2bfloat16_rn(-w[j]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_LOCAL, kLocal, !ok || *abort_flag)) break;
            if (tid == 0) {
                // stage st is free (its MMAs are done, copies read): prefetch m+2
                if (m + 2 < nchunks) issue_tma(m + 2);
                mbar_arrive(bar_ready);
            }
            if (m + 2 < nchunks) ++tma_issued[st];
            // ---- start the next chunk's D_kq ------------------------------------
            if (m + 1 < nchunks && !start_chunk(m + 1)) break;
        }
        // drain what this group launched, then report
        if (*abort_flag && tid == 0) {
            for (int s2 = 0; s2 < 2; ++s2)
                for (int i = tma_seen[s2]; i < tma_issued[s2]; ++i)
                    mbar_wait(&bar_tma[s2], (uint32_t)(i & 1), kWaitLimit);
            for (uint32_t i = bl_wait; i < bl_commit; ++i) mbar_wait(bar_l, i & 1, kWaitLimit);
        }
    } else {
        // ============================ state group ============================
        const int sq = warp & 3;  // TMEM lane quadrant = warp - 8
        const uint32_t lane_off = (uint32_t)(32 * sq) << 16;
        uint32_t bs_wait = 0, bs_commit = 0;
        for (int m = 0; m < nchunks; ++m) {
            const int st = m & 1;
            const long long t0 = t_begin + (long long)m * C;
            const int L = chunk_len(m);
            bool ok = wait_bar(bar_ready, (uint32_t)(m & 1), abort_flag);
            const float dec = hand_gc[st];  // read before the barrier: the slot is reused two chunks on
            tc_fence_after();
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            // ---- D_vp += [-W; gamma Q] S^T ----------------------------------------
            if (tid == kLocal) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < DK / 16; ++k)
                    mma_bf16(tmem + COL_VP + 64 * st,
                             desc_sw128(sbase + OFF_WQ + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024),
                             desc_sw128(sbase + OFF_SB + k * 2048, 16384, 1024), ID_KM, 1);
                mma_commit(bar_s);
                mma_commit(bar_wqfree);
            }
            ++bs_commit;
            ok &= wait_bar(bar_s, bs_wait & 1, abort_flag);
            ++bs_wait;
            tc_fence_after();
            // ---- V' = rows 0-63 as the MN-major operand --------------------------
            if (sq < 2) {
                float vp[64];
                tmem_load<64>(tmem + lane_off + COL_VP + 64 * st, vp);
                const int r = 32 * sq + lane;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    *reinterpret_cast<uint4 *>(sm + OFF_VP + sw128(r, j)) = pack8(vp + 8 * j);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            // ---- D_ds = K^^T V';  D_vp += [0; P] V' --------------------------------
            if (tid == kLocal) {
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_DS, desc_sw128(sbase + OFF_KH + k * 2048, 8192, 1024),
                             desc_sw128(sbase + OFF_VP + k * 2048, 8192, 1024), ID_MM, k > 0);
#pragma unroll
                for (int k = 0; k < C / 16; ++k)
                    mma_bf16(tmem + COL_VP + 64 * st, desc_sw128(sbase + OFF_Z + k * 32, 16, 1024),
                             desc_sw128(sbase + OFF_VP + k * 2048, 8192, 1024), ID_KM, 1);
                mma_commit(bar_s);
                mma_commit(bar_pfree);
            }
            ++bs_commit;
            ok &= wait_bar(bar_s, bs_wait & 1, abort_flag);
            ++bs_wait;
            tc_fence_after();
            // ---- S <- e^{g_C} S + dS;  output rows -------------------------------
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                float ds[32];
                tmem_load<32>(tmem + lane_off + COL_DS + 32 * hh, ds);  // lane c: dS[i][c]
#pragma unroll
                for (int i = 0; i < 32; ++i) s_reg[32 * hh + i] = dec * s_reg[32 * hh + i] + ds[i];
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                *reinterpret_cast<uint4 *>(sm + OFF_SB + sw128(c_st, j)) = pack8(s_reg + 8 * j);
            if (sq >= 2) {
                float o[64];
                tmem_load<64>(tmem + lane_off + COL_VP + 64 * st, o);
                const int r = 32 * (sq - 2) + lane;
                if (r < L) {
                    __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.o) +
                                         ((t0 + r) * H + h) * (long long)a.dv + v0;
#pragma unroll
                    for (int j = 0; j < 8; ++j) reinterpret_cast<uint4 *>(dst)[j] = pack8(o + 8 * j);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            if (named_bar_or(BAR_STATE, kState, !ok || *abort_flag)) break;
            if (tid == kLocal) mbar_arrive(&bar_vpfree[st]);
        }
        if (*abort_flag) {
            if (tid == kLocal)
                for (uint32_t i = bs_wait; i < bs_commit; ++i) mbar_wait(bar_s, i & 1, kWaitLimit);
        } else if (a.s_final) {
#pragma unroll
            for (int i = 0; i < DVS; ++i) a.s_final[st_base + (size_t)(v0 + i) * DK + c_st] = s_reg[i];
        }
    }

    tc_fence_before();
    __syncthreads();
    if (tid == 0 && *abort_flag) atomicOr(a.err, kErrTimeout);
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
