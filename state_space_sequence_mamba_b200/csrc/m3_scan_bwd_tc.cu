// Chunked backward of the prefill scan on the sm_100a tensor cores (bf16 operands, fp32
// accumulators in TMEM, fp32 state adjoint), for bf16 inputs with N = 128, P = 64 and rank
// R in {1, 2, 4, 8}: a chunk is 64 operand rows, Q = 64 / R tokens of R (token, rank) rows,
// as in the forward scan, and the token mask acts on full R x R blocks.
//
// Method ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.3
// eq. 7 for the chunk mask M = L1 . L2, Sec. 3.3 for the chunked algorithm, and the chain
// rule through it). With the forward's chunk quantities (cum = chunk-local inclusive sum of
// dt A, w_t = gamma_t + (1 - lam_{t+1}) dt_{t+1}, M[t,s] = e^{cum_t - cum_s} w_s for s < t,
// gamma_t on the diagonal, H0' the primed state before the chunk) and G_n the state adjoint
// dL/dh at the first token of the next chunk (the final state's gradient after the last
// chunk, with alpha_n = 1), each chunk needs:
//     S' = Bbar Cbar^T,  Z = X dY^T,  Q1 = Bbar G_n                 (tensor cores, M64)
//     Ps = M^T o S',  Pz = M^T o Z                                   (CUDA cores)
//     dx    = Ps dY + diag(w e^{cx_T - cum}) Q1                      (tensor cores, then Q1 scaled)
//     dBbar = Pz Cbar + diag(w e^{cx_T - cum}) X G_n^T               (tensor cores, N128)
//     dCbar = Pz^T Bbar + diag(e^{cum - cum_0}) dY (e^{cum_0} H0')^T (tensor cores, N128)
//     G_0   = Cbar^T diag(e^{cum - cum_0}) dY + e^{cx_T - cum_0} G_n (tensor cores, M128)
// where cx_T = cum_end + dt_n A_n (alpha_n = e^{dt_n A_n} of the next chunk's first token).
// The per-token scalars the step and trapezoid gradients need are row sums of the element-
// wise products of the two 64 x 64 matrices, summed over the token's rows:
//     dg_t = <G_t, u_t>     = sum_{s>=t} e^{cum_s - cum_t} S'[t,s] Z[t,s] + e^{cx_T - cum_t} q_t
//     db_{t+1} = <G_{t+1}, u_t> = sum_{s>t} e^{cum_s - cum_{t+1}} S'[t,s] Z[t,s]
//                                 + e^{cx_T - cum_{t+1}} q_t,     q_t = (Bbar_t G_n) . x_t
// The decay gradient D_t = <G_t, alpha_t h_{t-1}> is formed per chunk from sums that do not
// cancel (see the per-token term below), the angle adjoint dPhi_t (the cross products of
// dBbar and dCbar with Bbar and Cbar, summed from the end of the sequence) gives
// dtheta = dt dPhi. dBbar and dCbar are rotated back to the normalised, biased frame; the
// RMS-norm backward, the sum over the heads of a group and the step-scalar chain rule run in
// the kernels the sequential backward also uses.
//
// One CTA per (batch, head) unit walks its chunks from the last to the first, carrying G_n
// (fp32 in registers, bf16 as an operand) and the angle adjoint. The primed chunk-start
// states come from a forward state pass (the tensor-core scan's state-only form), which
// stores e^{cum_0} H0' per chunk in the swizzled bf16 operand layout and the angle before each
// chunk. Every sum has a fixed order: the gradients are reproducible run to run.
#include <cstdlib>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "m3_common.cuh"
#include "m3_internal.h"
#include "m3_sm100.cuh"

namespace m3 {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kN = 128, kP = 64, kHalf = 64, kQ = 64;   // kQ: operand rows per chunk
constexpr int kPhiStride = 68;   // floats per row of the angle tile (padded against conflicts)

// Shared memory (bytes from a 1024-byte aligned base). Operand tiles are 64 rows of 128 bytes
// per 64-column slab, 128-byte swizzled; 128-column tiles hold two slabs 8192 bytes apart.
constexpr uint32_t S_XT = 0;          // X [t][p] (TMA)
constexpr uint32_t S_DT = 8192;       // dY [t][p] (TMA)
constexpr uint32_t S_XS = 16384;      // diag(vn) X
constexpr uint32_t S_DS = 24576;      // diag(e^{cum - cum_0}) dY
constexpr uint32_t S_PS = 32768;      // Ps = M^T o S'
constexpr uint32_t S_PZ = 40960;      // Pz = M^T o Z
constexpr uint32_t S_BT = 49152;      // Bbar [t][n]
constexpr uint32_t S_BS = 65536;      // staging of the epilogue's rows (16 KB)
constexpr uint32_t S_CT = 81920;      // raw C (TMA), rotated in place to Cbar
constexpr uint32_t S_RB = 98304;      // raw B (TMA)
constexpr uint32_t S_GN = 114688;     // G_n bf16 [n][p], two buffers of 16384
constexpr uint32_t S_HS = 147456;     // e^{cum_0} H0' bf16 [n][p] (bulk copy)
constexpr uint32_t S_TH = 163840;     // theta [t][i] (TMA)
constexpr uint32_t SC_SLOT = 1152;   // room for [Q + 1 tokens][4 heads] fp32, Q <= 64
constexpr uint32_t S_SC = 172032;     // dt, A, lam boxes
constexpr uint32_t S_RS = S_SC + 3 * SC_SLOT;            // RMS scales, 64 float2
constexpr uint32_t S_PHI0 = S_RS + 512;                  // angle before the chunk, 64 floats
constexpr uint32_t S_PHI = S_PHI0 + 256;                 // angles, then angle adjoints [64][68]
constexpr uint32_t S_F = S_PHI + 64 * kPhiStride * 4;    // chunk scalars (floats, below)
constexpr uint32_t S_RED = S_F + 4 * 800;                // row partials [5 kinds][4 slots][64]
constexpr uint32_t S_CU = S_RED + 4 * 5 * 4 * 64;        // column partials [4 row blocks][64]
constexpr uint32_t S_TOK = S_CU + 4 * 4 * 64;            // per-token dg, db_{t+1}: [2][64]
constexpr uint32_t S_SEG = S_TOK + 4 * 2 * 64;           // angle walk: [8 segments][32] float2
constexpr uint32_t S_BIAS = S_SEG + 2048;                // bias_B, bias_C fp32 [2][R][128]
constexpr uint32_t S_SUF = S_BIAS + 8192;                // suffix-scan segment sums [4][64]
constexpr uint32_t S_CAR = S_SUF + 1024;                 // angle-adjoint carry [64]
constexpr uint32_t S_END = S_CAR + 256;
constexpr uint32_t kSmemBytes = S_END + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory");

// chunk scalars (float offsets into S_F)
constexpr int F_C2 = 0;      // [65] log2e * cum_t (t < Q), log2e * cx_T at [Q]
constexpr int F_GAM = 80;    // gamma_t
constexpr int F_W = 144;     // w_t
constexpr int F_VN = 208;    // w_t e^{cx_T - cum_t}
constexpr int F_EE = 272;    // e^{cx_T - cum_t}
constexpr int F_EB = 336;    // e^{cx_T - cum_{t+1}} (1 for the chunk's last token)
constexpr int F_DS = 400;    // e^{cum_t - cum_0}
constexpr int F_DT = 464;    // dt_t
constexpr int F_BETA = 528;  // [65] beta_t; beta of the next chunk's first token at [Q]
constexpr int F_MISC = 600;  // e^{cx_T - cum_0}, alpha_0, beta_0
// row-partial kinds
constexpr int R_KG = 0, R_KB = 1, R_Q = 2, R_RU = 3, R_V = 4;

// TMEM columns (512 allocated, one CTA per SM)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0;      // S', then dx
constexpr uint32_t T_Z = 64;     // Z, then Yo = Cbar (e^{cum_0} H0')
constexpr uint32_t T_Q = 128;    // Q1
constexpr uint32_t T_G = 192;    // G_0 (M128)
constexpr uint32_t T_DB = 256;   // dBbar (N128)
constexpr uint32_t T_DC = 384;   // dCbar (N128)

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}
// 16 consecutive bf16 of one swizzled row (cols c .. c + 15, c a multiple of 8) as fp32
__device__ __forceinline__ void load_row16(const uint8_t* tile, int row, int c, float (&v)[16]) {
    const uint4 a = *reinterpret_cast<const uint4*>(tile + swz128(row, c));
    const uint4 b = *reinterpret_cast<const uint4*>(tile + swz128(row, c + 8));
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float2 f = bf2_to_f2(w[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

// A [64 rows][64 fp32] staging tile: 16-byte chunk ch of row r at r * 256 + (ch ^ (r & 15)) * 16,
// so that 16 rows written at the same columns, or one row read whole, hit distinct banks.
__device__ __forceinline__ uint32_t staged_off(int row, int ch) {
    return static_cast<uint32_t>(row) * 256u + (static_cast<uint32_t>(ch ^ (row & 15)) << 4);
}
// 16 consecutive fp32 of row `row` starting at column c (a multiple of 4) into a staging tile
__device__ __forceinline__ void stage_row(uint8_t* tile, int row, int c, const float (&v)[16]) {
#pragma unroll
    for (int m = 0; m < 4; ++m)
        *reinterpret_cast<float4*>(tile + staged_off(row, c / 4 + m)) =
            make_float4(v[4 * m], v[4 * m + 1], v[4 * m + 2], v[4 * m + 3]);
}
// The same tile read as [64 rows][128 bf16]: columns c .. c + 15 from lo and 64 + c .. 79 + c
// from hi (c a multiple of 8), each rounded to bf16
__device__ __forceinline__ void stage_row_bf16(uint8_t* tile, int row, int c, const float (&lo)[16],
                                               const float (&hi)[16]) {
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        *reinterpret_cast<uint4*>(tile + staged_off(row, c / 8 + m)) =
            make_uint4(pack_bf16(lo[8 * m], lo[8 * m + 1]), pack_bf16(lo[8 * m + 2], lo[8 * m + 3]),
                       pack_bf16(lo[8 * m + 4], lo[8 * m + 5]), pack_bf16(lo[8 * m + 6], lo[8 * m + 7]));
        *reinterpret_cast<uint4*>(tile + staged_off(row, 8 + c / 8 + m)) =
            make_uint4(pack_bf16(hi[8 * m], hi[8 * m + 1]), pack_bf16(hi[8 * m + 2], hi[8 * m + 3]),
                       pack_bf16(hi[8 * m + 4], hi[8 * m + 5]), pack_bf16(hi[8 * m + 6], hi[8 * m + 7]));
    }
}

}  // namespace

struct BwdTcArgs {
    ScanParams p;
    const float2* rs;          // RMS scales [b][G][Lpad][R] (x: B, y: C), null without the norm
    const uint8_t* chunk_h;    // [units][nch][16384]: e^{cum_0} H0' bf16, swizzled [n][p]
    const float* chunk_phi;    // [units][nch][64]: the angle before each chunk
    const float* hfin;         // [units][N][P]: the final state
    const float* dh1;          // gradients of the final state (nullable)
    const float* dphi1;
    const float* dprevx1;
    float* dx;                 // [b, L, H, R, P]
    float* dtheta;             // [b, L, H, N/2]
    __nv_bfloat16* wdB;        // [b, L, H, R, N]: dBbar rotated back (per head), bf16
    __nv_bfloat16* wdC;
    float* wsc;                // [units][L][4]: db, dg, decay term, theta.dPhi per token
    float* wprev;              // [units][R][N]: the same for the initial state's previous B
    float* wF;                 // [units]: <dL/dh_final, h_final>
    float* wbias;              // [units][2][R][N]: this unit's bias sums (B, C)
    float* dh0;                // initial-state gradients (nullable)
    float* dphi0;
    float* dprevx0;
    int32_t* status;
    int nch;
};

struct BwdMaps {
    CUtensorMap x, dy, theta, B, C, dt, A, lam;
};

namespace {

// R: the rank; a chunk is Q = 64 / R tokens, its 64 operand rows are (token, rank) pairs,
// row = token * R + rank, and the token mask acts on full R x R blocks.
template <int R, bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
bwd_tc_kernel(const BwdTcArgs a, const __grid_constant__ BwdMaps maps) {
    constexpr int Q = kQ / R;                      // tokens per chunk
    constexpr uint32_t SC_ONE = (Q + 1) * 16;      // bytes of one scalar box
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const ScanParams& p = a.p;
    float* sf = reinterpret_cast<float*>(sm + S_F);
    float* red = reinterpret_cast<float*>(sm + S_RED);
    float2* s_seg = reinterpret_cast<float2*>(sm + S_SEG);
    float* s_bias = reinterpret_cast<float*>(sm + S_BIAS);
    float* s_suf = reinterpret_cast<float*>(sm + S_SUF);
    float* s_car = reinterpret_cast<float*>(sm + S_CAR);
    float* s_cu = reinterpret_cast<float*>(sm + S_CU);
    float* s_tok = reinterpret_cast<float*>(sm + S_TOK);
    float* sphi = reinterpret_cast<float*>(sm + S_PHI);
    // loads in four groups, each issued as soon as the previous chunk has released its buffers:
    // A (scalar boxes, raw B, RMS scales, the chunk's start angle), X, H (the chunk-start state),
    // B (theta, dY, raw C)
    __shared__ uint64_t bar_a, bar_x, bar_h, bar_b, bar_m1, bar_g, bar_m2;
    __shared__ uint32_t tslot;
    __shared__ int s_abort;
    __shared__ int s_cnt[4];   // MMA groups m1, g, m2 committed (index 1..3)
    __shared__ int s_lcnt[4];  // load groups A, X, H, B issued
    __shared__ float s_wred[8];
    __shared__ float s_t4[8];
    __shared__ float s_dnext;   // D'_t of the first token of the chunk after the current one

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, wh = warp >> 2;
    const int64_t u = blockIdx.x, bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int L = static_cast<int>(p.L), nch = a.nch;
    const int ib = static_cast<int>(bb), ih = static_cast<int>(hh), ig = static_cast<int>(g);
    const int hc = ih & 3;
    const int64_t H = p.H;
    const int64_t Lpad = static_cast<int64_t>(nch) * Q;
    const float dtb = (kRaw && p.dt_bias) ? p.dt_bias[hh] : 0.f;
    const bool zoh = kRaw && (p.flags & M3_DISC_ZOH);
    const float2* rsu = a.rs ? a.rs + (bb * p.G + g) * Lpad * R : nullptr;

    auto issue_a = [&](int c) {
        const int t0 = c * Q;
        mbar_arrive_expect_tx(&bar_a, 3 * SC_ONE + 16384 + (rsu ? 512u : 0u) + 256);
        const int h4 = ih & ~3;
        tma_load_3d(sm + S_SC, &maps.dt, &bar_a, h4, t0, ib);
        tma_load_3d(sm + S_SC + SC_SLOT, &maps.A, &bar_a, h4, t0, ib);
        tma_load_3d(sm + S_SC + 2 * SC_SLOT, &maps.lam, &bar_a, h4, t0, ib);
        tma_load_5d(sm + S_RB, &maps.B, &bar_a, 0, 0, ig, t0, ib);
        tma_load_5d(sm + S_RB + 8192, &maps.B, &bar_a, kHalf, 0, ig, t0, ib);
        if (rsu) bulk_load(sm + S_RS, rsu + static_cast<int64_t>(t0) * R, 512u, &bar_a);
        bulk_load(sm + S_PHI0, a.chunk_phi + (u * nch + c) * kHalf, 256u, &bar_a);
        s_lcnt[0] += 1;
    };
    auto issue_x = [&](int c) {
        mbar_arrive_expect_tx(&bar_x, 8192);
        tma_load_5d(sm + S_XT, &maps.x, &bar_x, 0, 0, ih, c * Q, ib);
        s_lcnt[1] += 1;
    };
    auto issue_h = [&](int c) {
        mbar_arrive_expect_tx(&bar_h, 16384);
        bulk_load(sm + S_HS, a.chunk_h + (u * nch + c) * 16384, 16384u, &bar_h);
        s_lcnt[2] += 1;
    };
    auto issue_b = [&](int c) {
        // test hook: CTA 0 skips this group for the chunk it reaches at step test_skip_theta,
        // so that its bounded wait runs out (a load that nothing issues)
        if (blockIdx.x == 0 && p.test_skip_theta > 0 && c == nch - 1 - p.test_skip_theta) return;
        const int t0 = c * Q;
        mbar_arrive_expect_tx(&bar_b, Q * 128 + 8192 + 16384);
        tma_load_4d(sm + S_TH, &maps.theta, &bar_b, 0, ih, t0, ib);
        tma_load_5d(sm + S_DT, &maps.dy, &bar_b, 0, 0, ih, t0, ib);
        tma_load_5d(sm + S_CT, &maps.C, &bar_b, 0, 0, ig, t0, ib);
        tma_load_5d(sm + S_CT + 8192, &maps.C, &bar_b, kHalf, 0, ig, t0, ib);
        s_lcnt[3] += 1;
    };

    // ---------------- set-up ----------------
    if (tid == 0) {
        mbar_init(&bar_a, 1);
        mbar_init(&bar_x, 1);
        mbar_init(&bar_h, 1);
        mbar_init(&bar_b, 1);
        mbar_init(&bar_m1, 1);
        mbar_init(&bar_g, 1);
        mbar_init(&bar_m2, 1);
        fence_mbar_init();
        s_abort = 0;
        s_cnt[0] = s_cnt[1] = s_cnt[2] = s_cnt[3] = 0;
        s_lcnt[0] = s_lcnt[1] = s_lcnt[2] = s_lcnt[3] = 0;
        if (nch > 0) {
            issue_a(nch - 1);
            issue_b(nch - 1);
            issue_x(nch - 1);
            issue_h(nch - 1);
        }
    }
    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    for (int i = tid; i < 2 * R * kN; i += kThreads) {
        const float* bsrc = i < R * kN ? p.Bbias : p.Cbias;
        s_bias[i] = bsrc ? bsrc[hh * R * kN + (i % (R * kN))] : 0.f;
    }
    if (tid < kHalf) s_car[tid] = a.dphi1 ? a.dphi1[u * kHalf + tid] : 0.f;

    // G_n = dL/dh_final in registers: row n = 32 q4 + lane, columns [32 wh, 32 wh + 32); and
    // <dL/dh_final, h_final> for the decay gradient
    const int nrow = 32 * q4 + lane;
    float gr[32];
    {
        float f = 0.f;
        const float4* gsrc = a.dh1 ? reinterpret_cast<const float4*>(a.dh1 + (u * kN + nrow) * kP + 32 * wh) : nullptr;
        const float4* hsrc = reinterpret_cast<const float4*>(a.hfin + (u * kN + nrow) * kP + 32 * wh);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = gsrc ? gsrc[j] : make_float4(0.f, 0.f, 0.f, 0.f);
            gr[4 * j] = v.x; gr[4 * j + 1] = v.y; gr[4 * j + 2] = v.z; gr[4 * j + 3] = v.w;
            if (gsrc) {
                const float4 h = hsrc[j];
                f = fmaf(v.x, h.x, fmaf(v.y, h.y, fmaf(v.z, h.z, fmaf(v.w, h.w, f))));
            }
        }
        f = warp_sum(f);
        if (lane == 0) s_wred[warp] = f;
    }
    auto store_gn = [&](int buf) {
        uint8_t* dst = sm + S_GN + buf * 16384;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v;
            v.x = pack_bf16(gr[8 * i + 0], gr[8 * i + 1]);
            v.y = pack_bf16(gr[8 * i + 2], gr[8 * i + 3]);
            v.z = pack_bf16(gr[8 * i + 4], gr[8 * i + 5]);
            v.w = pack_bf16(gr[8 * i + 6], gr[8 * i + 7]);
            *reinterpret_cast<uint4*>(dst + swz128(nrow, 32 * wh + 8 * i)) = v;
        }
    };
    store_gn(0);
    fence_proxy_async();
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (tid == 0) {
        float f = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) f += s_wred[w];
        a.wF[u] = f;
        s_dnext = f;   // D_L = <dL/dh_final, h_final>
    }
    const uint32_t tmem = tslot;
    const uint32_t lanebase = (32u * q4) << 16;

    // per-thread bias sums over the rows this thread owns in every chunk (row = 16 q4 +
    // lane % 16, always of rank row % R; B and C columns col0 + k and col0 + 64 + k, k < 16)
    float accB[32], accC[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) accB[k] = accC[k] = 0.f;

    const int trow = 16 * q4 + (lane & 15);
    const int col0 = 16 * wh + ((lane >> 4) ? 32 : 0);
    const int slot = 2 * wh + (lane >> 4);
    const uint32_t aXT = smem_u32(sm + S_XT), aDT = smem_u32(sm + S_DT);
    const uint32_t aXS = smem_u32(sm + S_XS), aDS = smem_u32(sm + S_DS);
    const uint32_t aPS = smem_u32(sm + S_PS), aPZ = smem_u32(sm + S_PZ);
    const uint32_t aBT = smem_u32(sm + S_BT);
    const uint32_t aCT = smem_u32(sm + S_CT), aHS = smem_u32(sm + S_HS);
    const uint32_t aGN = smem_u32(sm + S_GN);

    for (int it = 0; it < nch; ++it) {
        const int c = nch - 1 - it;
        const int cur = it & 1;
        const uint32_t par = static_cast<uint32_t>(it & 1);
        const int t0 = c * Q;
        const int T = (L - t0) < Q ? (L - t0) : Q;   // tokens of this chunk
        if (!mbar_wait(&bar_a, par)) s_abort = 1;   // scalar boxes, raw B, scales, start angle
        if constexpr (kRaw) {
            // this head's column of the dt and lam boxes: softplus / sigmoid in place
            float* sSc = reinterpret_cast<float*>(sm + S_SC);
            for (int i = tid; i < 2 * (Q + 1); i += kThreads) {
                const int t = i <= Q ? i : i - (Q + 1);
                if (t0 + t >= L) continue;
                if (i <= Q) {
                    float* d = sSc + t * 4 + hc;
                    *d = step_dt<true>(*d, dtb, p.flags);
                } else {
                    float* lm = sSc + 2 * SC_SLOT / 4 + t * 4 + hc;
                    *lm = step_lam<true>(*lm, p.flags);
                }
            }
            __syncthreads();
        }
        // ---- chunk scalars (warp 0) ----
        if (warp == 0) {
            const float* sSc = reinterpret_cast<const float*>(sm + S_SC);
            constexpr int oA = SC_SLOT / 4, oL = 2 * SC_SLOT / 4;
            float av[2], dv[2], gv[2], wv[2], bv[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                av[k] = dv[k] = gv[k] = wv[k] = bv[k] = 0.f;
                if (t < T) {
                    const float d = sSc[t * 4 + hc], A = sSc[oA + t * 4 + hc];
                    const float lm = sSc[oL + t * 4 + hc];
                    dv[k] = d;
                    av[k] = d * A;
                    gv[k] = zoh ? zoh_gamma(d, A) : lm * d;
                    bv[k] = zoh ? 0.f : (1.f - lm) * d * __expf(d * A);
                    const float cn = zoh ? 0.f : (1.f - sSc[oL + (t + 1) * 4 + hc]) * sSc[(t + 1) * 4 + hc];
                    wv[k] = gv[k] + cn;
                }
            }
            const float s0 = warp_inclusive_scan(av[0]);
            const float tot0 = __shfl_sync(0xffffffffu, s0, 31);
            const float s1 = warp_inclusive_scan(av[1]) + tot0;
            const float cum_end = __shfl_sync(0xffffffffu, s1, 31);   // padded tokens add 0
            const float a_next = sSc[Q * 4 + hc] * sSc[oA + Q * 4 + hc];   // 0 past the end
            const float cxT = cum_end + a_next;
            const float cum0 = __shfl_sync(0xffffffffu, s0, 0);
            // cum_{t+1} for every t (cx_T after the chunk's last real token)
            const float n0 = __shfl_down_sync(0xffffffffu, s0, 1);
            const float n1 = __shfl_down_sync(0xffffffffu, s1, 1);
            const float s1first = __shfl_sync(0xffffffffu, s1, 0);
            constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                const float cm = k ? s1 : s0;
                float cnext = k ? n1 : (lane == 31 ? s1first : n0);
                if (t + 1 >= T) cnext = cxT;
                const bool real = t < T;
                sf[F_C2 + t] = cm * kLog2e;
                sf[F_GAM + t] = gv[k];
                sf[F_W + t] = wv[k];
                sf[F_VN + t] = real ? wv[k] * __expf(cxT - cm) : 0.f;
                sf[F_EE + t] = real ? __expf(cxT - cm) : 0.f;
                sf[F_EB + t] = real ? __expf(cxT - cnext) : 0.f;
                sf[F_DS + t] = real ? __expf(cm - cum0) : 0.f;
                sf[F_DT + t] = dv[k];
                sf[F_BETA + t] = bv[k];
            }
            __syncwarp();
            if (lane == 0) {
                sf[F_C2 + Q] = cxT * kLog2e;
                sf[F_BETA + Q] = zoh ? 0.f
                    : (1.f - sSc[oL + Q * 4 + hc]) * sSc[Q * 4 + hc] * __expf(a_next);
                sf[F_MISC + 0] = __expf(cxT - cum0);
                sf[F_MISC + 1] = __expf(cum0);
                const float d0 = sSc[hc], l0 = sSc[oL + hc];
                sf[F_MISC + 2] = zoh ? 0.f : (1.f - l0) * d0 * __expf(cum0);
            }
        }
        __syncthreads();

        // ---- angles of the chunk and the rotation of B and C (warp = 8 tokens, lane = pair
        // couple (2 lane, 2 lane + 1), partners + N/2) ----
        if (!mbar_wait(&bar_b, par)) s_abort = 1;   // theta, dY, raw C
        {
            const int jp = 2 * lane;
            constexpr int TPS = Q / 8;   // tokens per warp
            const float* phi0 = reinterpret_cast<const float*>(sm + S_PHI0);
            float inc[TPS][2];
            float sum0 = 0.f, sum1 = 0.f;
#pragma unroll
            for (int k = 0; k < TPS; ++k) {
                const int t = warp * TPS + k;
                const uint32_t th = *reinterpret_cast<const uint32_t*>(sm + S_TH + swz128(t, jp));
                const float dd = sf[F_DT + t];
                inc[k][0] = dd * __uint_as_float(th << 16);
                inc[k][1] = dd * __uint_as_float(th & 0xFFFF0000u);
                sum0 += inc[k][0];
                sum1 += inc[k][1];
            }
            s_seg[warp * 32 + lane] = make_float2(sum0, sum1);
            __syncthreads();
            float a0 = reduce_2pi(phi0[jp]), a1 = reduce_2pi(phi0[jp + 1]);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float2 v = s_seg[k * 32 + lane];
                if (k < warp) { a0 += v.x; a1 += v.y; }
            }
#pragma unroll
            for (int k = 0; k < TPS; ++k) {
                const int t = warp * TPS + k;
                a0 += inc[k][0];
                a1 += inc[k][1];
                *reinterpret_cast<float2*>(sphi + t * kPhiStride + jp) = make_float2(a0, a1);
                float2 cs, sn;
                __sincosf(a0, &sn.x, &cs.x);
                __sincosf(a1, &sn.y, &cs.y);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                const int row = t * R + r;
                const float2 bB0 = *reinterpret_cast<const float2*>(s_bias + r * kN + jp);
                const float2 bB1 = *reinterpret_cast<const float2*>(s_bias + r * kN + jp + kHalf);
                const float2 bC0 = *reinterpret_cast<const float2*>(s_bias + (R + r) * kN + jp);
                const float2 bC1 = *reinterpret_cast<const float2*>(s_bias + (R + r) * kN + jp + kHalf);
                const float2 rs = (rsu && t < T) ? reinterpret_cast<const float2*>(sm + S_RS)[row]
                                                 : make_float2(1.f, 1.f);
                const uint32_t o = swz128(row, jp);
                {   // B: u = rs raw + bias, Bbar = (u0 c + u1 s, u1 c - u0 s)
                    const float2 r0 = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + S_RB + o));
                    const float2 r1 = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + S_RB + 8192 + o));
                    const float2 u0 = make_float2(fmaf(r0.x, rs.x, bB0.x), fmaf(r0.y, rs.x, bB0.y));
                    const float2 u1 = make_float2(fmaf(r1.x, rs.x, bB1.x), fmaf(r1.y, rs.x, bB1.y));
                    const float2 v0 = make_float2(fmaf(u0.x, cs.x, u1.x * sn.x), fmaf(u0.y, cs.y, u1.y * sn.y));
                    const float2 v1 = make_float2(fmaf(u1.x, cs.x, -u0.x * sn.x), fmaf(u1.y, cs.y, -u0.y * sn.y));
                    *reinterpret_cast<uint32_t*>(sm + S_BT + o) = pack_bf16(v0.x, v0.y);
                    *reinterpret_cast<uint32_t*>(sm + S_BT + 8192 + o) = pack_bf16(v1.x, v1.y);
                }
                {   // C, in place
                    const float2 r0 = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + S_CT + o));
                    const float2 r1 = bf2_to_f2(*reinterpret_cast<const uint32_t*>(sm + S_CT + 8192 + o));
                    const float2 u0 = make_float2(fmaf(r0.x, rs.y, bC0.x), fmaf(r0.y, rs.y, bC0.y));
                    const float2 u1 = make_float2(fmaf(r1.x, rs.y, bC1.x), fmaf(r1.y, rs.y, bC1.y));
                    *reinterpret_cast<uint32_t*>(sm + S_CT + o) =
                        pack_bf16(fmaf(u0.x, cs.x, u1.x * sn.x), fmaf(u0.y, cs.y, u1.y * sn.y));
                    *reinterpret_cast<uint32_t*>(sm + S_CT + 8192 + o) =
                        pack_bf16(fmaf(u1.x, cs.x, -u0.x * sn.x), fmaf(u1.y, cs.y, -u0.y * sn.y));
                }
                }
            }
        }
        // ---- Xs = diag(vn) X and Ds = diag(e^{cum - cum_0}) dY (rows keep their swizzle) ----
        if (!mbar_wait(&bar_x, par)) s_abort = 1;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int e = tid + i * kThreads;
            const int row = e >> 3, ch = e & 7;
            const uint32_t o = static_cast<uint32_t>(row) * 128u + (static_cast<uint32_t>(ch) << 4);
            const float fx = sf[F_VN + row / R], fd = sf[F_DS + row / R];
            const uint4 vx = *reinterpret_cast<const uint4*>(sm + S_XT + o);
            const uint4 vd = *reinterpret_cast<const uint4*>(sm + S_DT + o);
            const uint32_t wx[4] = {vx.x, vx.y, vx.z, vx.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
            uint32_t ox[4], od[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 x2 = bf2_to_f2(wx[j]), d2 = bf2_to_f2(wd[j]);
                ox[j] = pack_bf16(fx * x2.x, fx * x2.y);
                od[j] = pack_bf16(fd * d2.x, fd * d2.y);
            }
            *reinterpret_cast<uint4*>(sm + S_XS + o) = make_uint4(ox[0], ox[1], ox[2], ox[3]);
            *reinterpret_cast<uint4*>(sm + S_DS + o) = make_uint4(od[0], od[1], od[2], od[3]);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;

        // ---- S', Z, Q1 and G_0 on the tensor cores ----
        if (tid == 0) {
            constexpr uint32_t hi = desc_hi_sw128(1024);
            const uint32_t idS = idesc_bf16(64, 64, false, false);
            const uint32_t idQ = idesc_bf16(64, 64, false, true);
            const uint32_t idG = idesc_bf16(128, 64, true, true);
            const uint32_t loB = desc_lo(aBT, 16), loC = desc_lo(aCT, 16);
            const uint32_t loX = desc_lo(aXT, 16), loD = desc_lo(aDT, 16);
            const uint32_t loGn = desc_lo(aGN + cur * 16384, 16384);
            const uint32_t loCt = desc_lo(aCT, 8192), loDS = desc_lo(aDS, 8192);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tmem + T_S, desc_pack(loB + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loC + (kmajor_off(k, 8192) >> 4), hi), idS, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_Z, desc_pack(loX + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loD + (kmajor_off(k, 8192) >> 4), hi), idS, k > 0);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tmem + T_Q, desc_pack(loB + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loGn + (mnmajor_off(k) >> 4), hi), idQ, k > 0);
            mma_commit(smem_u32(&bar_m1));
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_G, desc_pack(loCt + (mnmajor_off(k) >> 4), hi),
                         desc_pack(loDS + (mnmajor_off(k) >> 4), hi), idG, k > 0);
            mma_commit(smem_u32(&bar_g));
            s_cnt[1] += 1;
            s_cnt[2] += 1;
            // the rotation and the scalars have read their inputs: the earlier chunk's group A
            if (c > 0) issue_a(c - 1);
        }
        __syncwarp();

        // ---- Ps, Pz and the row sums from S', Z, Q1 ----
        {
            if (!mbar_wait(&bar_m1, par)) s_abort = 1;
            fence_after_sync();
            float sv[16], zv[16], qv[16];
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_S + 16u * wh, sv);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_Z + 16u * wh, zv);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_Q + 16u * wh, qv);
            const int t = trow;                 // operand row
            const int tt = t / R;               // its token
            const float c2t = sf[F_C2 + tt], c2t1 = sf[F_C2 + tt + 1];
            const float wt = sf[F_W + tt], gt = sf[F_GAM + tt];
            float xv[16];
            load_row16(sm + S_XT, t, col0, xv);
            tmem_wait_ld();
            // e^{cum_s - cum_t} = e^{cum_s - cum_{t+1}} alpha_{t+1}: one exponential per element,
            // both factors <= 1; the selects keep the warp on one path
            const float alpha1 = ex2_approx(fminf(c2t1 - c2t, 0.f));
            float kg = 0.f, kb = 0.f, qq = 0.f, ru = 0.f;
            float cu[16];
            uint32_t ps[8], pz[8];
#pragma unroll
            for (int j = 0; j < 16; j += 2) {
                float pv[2], zz[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int s = (col0 + j + e) / R;   // the column's token
                    const float spv = sv[j + e], zvv = zv[j + e];
                    const bool after = s > tt, same = s == tt;   // same: the token's R x R block
                    const float fb = ex2_approx(fminf(sf[F_C2 + s] - c2t1, 0.f));
                    const float f = after ? fb * alpha1 : (same ? 1.f : 0.f);
                    const float m = after ? f * wt : (same ? gt : 0.f);
                    const float sz = spv * zvv;
                    kg = fmaf(f, sz, kg);
                    kb = fmaf(after ? fb : 0.f, sz, kb);
                    cu[j + e] = after ? m * sz : 0.f;   // the pair crosses every token in (tt, s]
                    ru += cu[j + e];
                    pv[e] = m * spv;
                    zz[e] = m * zvv;
                }
                ps[j / 2] = pack_bf16(pv[0], pv[1]);
                pz[j / 2] = pack_bf16(zz[0], zz[1]);
                qq = fmaf(qv[j], xv[j], fmaf(qv[j + 1], xv[j + 1], qq));
            }
            *reinterpret_cast<uint4*>(sm + S_PS + swz128(t, col0)) = make_uint4(ps[0], ps[1], ps[2], ps[3]);
            *reinterpret_cast<uint4*>(sm + S_PS + swz128(t, col0 + 8)) = make_uint4(ps[4], ps[5], ps[6], ps[7]);
            *reinterpret_cast<uint4*>(sm + S_PZ + swz128(t, col0)) = make_uint4(pz[0], pz[1], pz[2], pz[3]);
            *reinterpret_cast<uint4*>(sm + S_PZ + swz128(t, col0 + 8)) = make_uint4(pz[4], pz[5], pz[6], pz[7]);
            red[(R_KG * 4 + slot) * 64 + t] = kg;
            red[(R_KB * 4 + slot) * 64 + t] = kb;
            red[(R_Q * 4 + slot) * 64 + t] = qq;
            red[(R_RU * 4 + slot) * 64 + t] = ru;
            // column sums over the 16 rows of this half-warp, halving the list at each step
            // (lane bit 3 first); lane l & 15 then holds column col0 + (bit-reversed order)
            {
                float c8[8], c4[4], c2[2];
                bool up = lane & 8;
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    c8[j] = (up ? cu[j + 8] : cu[j]) + __shfl_xor_sync(0xffffffffu, up ? cu[j] : cu[j + 8], 8);
                up = lane & 4;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    c4[j] = (up ? c8[j + 4] : c8[j]) + __shfl_xor_sync(0xffffffffu, up ? c8[j] : c8[j + 4], 4);
                up = lane & 2;
#pragma unroll
                for (int j = 0; j < 2; ++j)
                    c2[j] = (up ? c4[j + 2] : c4[j]) + __shfl_xor_sync(0xffffffffu, up ? c4[j] : c4[j + 2], 2);
                up = lane & 1;
                const float c1 = (up ? c2[1] : c2[0]) + __shfl_xor_sync(0xffffffffu, up ? c2[0] : c2[1], 1);
                const int col = col0 + ((lane & 8) ? 8 : 0) + ((lane & 4) ? 4 : 0) + ((lane & 2) ? 2 : 0) +
                                ((lane & 1) ? 1 : 0);
                s_cu[q4 * 64 + col] = c1;
            }
        }
        // ---- G_0 = Cbar^T Ds + e^{cx_T - cum_0} G_n: the next (earlier) chunk's G_n ----
        if (!mbar_wait(&bar_h, par)) s_abort = 1;   // e^{cum_0} H0'
        {   // before G_n is replaced
            // <G_n, e^{cum_0} H0'> (this thread's 32 elements; summed per warp)
            float t4 = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 hv = *reinterpret_cast<const uint4*>(sm + S_HS + swz128(nrow, 32 * wh + 8 * i));
                const uint32_t hw[4] = {hv.x, hv.y, hv.z, hv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = bf2_to_f2(hw[j]);
                    t4 = fmaf(gr[8 * i + 2 * j], f.x, fmaf(gr[8 * i + 2 * j + 1], f.y, t4));
                }
            }
            t4 = warp_sum(t4);
            if (lane == 0) s_t4[warp] = t4;
        }
        {
            if (!mbar_wait(&bar_g, par)) s_abort = 1;
            fence_after_sync();
            const float e = sf[F_MISC + 0];
            const uint32_t ta = tmem + lanebase + T_G + 32u * wh;
            float d0[16], d1[16];
            tmem_ld_32x32b_x16(ta, d0);
            tmem_ld_32x32b_x16(ta + 16, d1);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                gr[j] = fmaf(e, gr[j], d0[j]);
                gr[16 + j] = fmaf(e, gr[16 + j], d1[j]);
            }
            store_gn(cur ^ 1);
        }
        fence_proxy_async();
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;

        // ---- dx, dBbar, dCbar on the tensor cores ----
        if (tid == 0) {
            constexpr uint32_t hi = desc_hi_sw128(1024);
            const uint32_t id64 = idesc_bf16(64, 64, false, true);
            const uint32_t idKN = idesc_bf16(64, 128, false, true);    // A K-major, B MN-major
            const uint32_t idKK = idesc_bf16(64, 128, false, false);   // both K-major
            const uint32_t idMN = idesc_bf16(64, 128, true, true);     // both MN-major
            const uint32_t loPS = desc_lo(aPS, 16), loPZ = desc_lo(aPZ, 16);
            const uint32_t loPZt = desc_lo(aPZ, 8192);
            const uint32_t loDTm = desc_lo(aDT, 8192);
            const uint32_t loXS = desc_lo(aXS, 16), loDS = desc_lo(aDS, 16);
            const uint32_t loGk = desc_lo(aGN + cur * 16384, 16);
            const uint32_t loHk = desc_lo(aHS, 16);
            const uint32_t loCt = desc_lo(aCT, 8192), loBt = desc_lo(aBT, 8192);
            const uint32_t loC2 = desc_lo(aCT, 16);
            // dx = Ps dY (+ diag(vn) Bbar G_n from the Q1 accumulator in the epilogue)
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_S, desc_pack(loPS + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loDTm + (mnmajor_off(k) >> 4), hi), id64, k > 0);
            // dBbar = Pz Cbar + Xs G_n^T
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_DB, desc_pack(loPZ + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loCt + (mnmajor_off(k) >> 4), hi), idKN, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_DB, desc_pack(loXS + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loGk + (kmajor_off(k, 16384) >> 4), hi), idKK, 1);
            // dCbar = Pz^T Bbar + Ds (e^{cum_0} H0')^T
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_DC, desc_pack(loPZt + (mnmajor_off(k) >> 4), hi),
                         desc_pack(loBt + (mnmajor_off(k) >> 4), hi), idMN, k > 0);
#pragma unroll
            for (int k = 0; k < 4; ++k)
                mma_bf16(tmem + T_DC, desc_pack(loDS + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loHk + (kmajor_off(k, 16384) >> 4), hi), idKK, 1);
            // Yo = Cbar (e^{cum_0} H0'), for the decay gradient's state term
            const uint32_t loHm = desc_lo(aHS, 16384);
#pragma unroll
            for (int k = 0; k < 8; ++k)
                mma_bf16(tmem + T_Z, desc_pack(loC2 + (kmajor_off(k, 8192) >> 4), hi),
                         desc_pack(loHm + (mnmajor_off(k) >> 4), hi), id64, k > 0);
            mma_commit(smem_u32(&bar_m2));
            s_cnt[3] += 1;
            if (c > 0) issue_x(c - 1);   // X was last read by Z, Xs and the q sums
        }
        __syncwarp();
        // per-token dg and the next token's db (one thread per token, fixed summation order
        // over the token's rows and the row partials)
        if (tid < Q) {
            const int t = tid;
            float kg = 0.f, kb = 0.f, q = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int s = 0; s < 4; ++s) {
                    kg += red[(R_KG * 4 + s) * 64 + t * R + r];
                    kb += red[(R_KB * 4 + s) * 64 + t * R + r];
                    q += red[(R_Q * 4 + s) * 64 + t * R + r];
                }
            const float dg = fmaf(sf[F_EE + t], q, kg), db1 = fmaf(sf[F_EB + t], q, kb);
            s_tok[t] = dg;
            s_tok[64 + t] = db1;
            if (t < T) {
                float* w = a.wsc + (u * L + t0 + t) * 4;
                w[1] = dg;
                if (t0 + t + 1 < L) w[4] = db1;
            }
        }

        // ---- epilogue: dx, dBbar and dCbar rotated back, the angle adjoint, dy . y ----
        {
            if (!mbar_wait(&bar_m2, par)) s_abort = 1;
            fence_after_sync();
            if (tid == 0 && c > 0) issue_h(c - 1);   // its readers (T4, dCbar, Yo) are done
            {   // theta into the Ps buffer (read by dx, done): its own buffer takes the next load
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int e = tid + i * kThreads;
                    *reinterpret_cast<uint4*>(sm + S_PS + 16 * e) =
                        *reinterpret_cast<const uint4*>(sm + S_TH + 16 * e);
                }
            }
            const int t = trow;                 // operand row
            const int tt = t / R, rk = t % R;   // its token and rank
            const bool real = tt < T;
            const int64_t tok = static_cast<int64_t>(t0) + tt;
            float vx[16], vb0[16], vb1[16], vc0[16], vc1[16];
            {
                float yo[16], dyv[16];
                tmem_ld_16x32bx2_x16(tmem + lanebase + T_Z + 16u * wh, yo);
                load_row16(sm + S_DT, t, col0, dyv);
                tmem_wait_ld();
                float v = 0.f;
#pragma unroll
                for (int k = 0; k < 16; ++k) v = fmaf(yo[k], dyv[k], v);
                red[(R_V * 4 + slot) * 64 + t] = v;
            }
            {   // dx = Ps dY + vn (Bbar G_n): the boundary term is Q1, still in TMEM, scaled
                float q1[16];
                tmem_ld_16x32bx2_x16(tmem + lanebase + T_S + 16u * wh, vx);
                tmem_ld_16x32bx2_x16(tmem + lanebase + T_Q + 16u * wh, q1);
                tmem_wait_ld();
                const float vn = sf[F_VN + tt];
#pragma unroll
                for (int k = 0; k < 16; ++k) vx[k] = fmaf(vn, q1[k], vx[k]);
            }
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_DB + 16u * wh, vb0);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_DB + 64u + 16u * wh, vb1);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_DC + 16u * wh, vc0);
            tmem_ld_16x32bx2_x16(tmem + lanebase + T_DC + 64u + 16u * wh, vc1);
            float bbar0[16], bbar1[16], cbar0[16], cbar1[16];
            load_row16(sm + S_BT, t, col0, bbar0);
            load_row16(sm + S_BT + 8192, t, col0, bbar1);
            load_row16(sm + S_CT, t, col0, cbar0);
            load_row16(sm + S_CT + 8192, t, col0, cbar1);
            tmem_wait_ld();
            float nb0[16], nb1[16], nc0[16], nc1[16];
            // the token's angles; with R > 1 the token's R rows sit in consecutive lanes, which
            // all read them before the sum of their angle adjoints replaces them
            float* ph = sphi + tt * kPhiStride + col0;
            float phv[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) phv[k] = ph[k];
            if constexpr (R > 1) __syncwarp();
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                float sn, cs;
                __sincosf(phv[k], &sn, &cs);
                const float db0 = vb0[k], db1 = vb1[k], dc0 = vc0[k], dc1 = vc1[k];
                nb0[k] = fmaf(db0, cs, -db1 * sn);
                nb1[k] = fmaf(db0, sn, db1 * cs);
                nc0[k] = fmaf(dc0, cs, -dc1 * sn);
                nc1[k] = fmaf(dc0, sn, dc1 * cs);
                float dl = fmaf(db0, bbar1[k], -db1 * bbar0[k]);
                dl = fmaf(dc0, cbar1[k], fmaf(-dc1, cbar0[k], dl));
#pragma unroll
                for (int o = 1; o < R; o <<= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
                if (rk == 0) ph[k] = real ? dl : 0.f;
            }
            if (real) {
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    accB[k] += nb0[k]; accB[16 + k] += nb1[k];
                    accC[k] += nc0[k]; accC[16 + k] += nc1[k];
                }
                if (a.dprevx1 && tok == L - 1) {
                    const float* px = a.dprevx1 + (u * R + rk) * kP + col0;
#pragma unroll
                    for (int k = 0; k < 16; ++k) vx[k] += px[k];
                }
            }
            // The rows go out through shared memory so that each half-warp stores one whole
            // 256-byte row (a thread holds 64 bytes of one row, 16 rows per half-warp), in the
            // buffers of Xs/Ds, Bs and this chunk's G_n operand, whose readers have finished:
            // dx in fp32, and the per-head dBbar and dCbar rows in bf16 (only their sums over
            // the group's heads are used, by the norm kernel).
            stage_row(sm + S_XS, t, col0, vx);
            stage_row_bf16(sm + S_BS, t, col0, nb0, nb1);
            stage_row_bf16(sm + S_GN + cur * 16384, t, col0, nc0, nc1);
            __syncthreads();
            for (int e = tid; e < 3 * 64 * 16; e += kThreads) {
                const int tile = e >> 10, row = (e >> 4) & 63, ch = e & 15;
                if (row / R >= T) continue;
                const int64_t grow = ((bb * L + t0 + row / R) * H + hh) * R + row % R;
                const uint8_t* src = tile == 0 ? sm + S_XS : tile == 1 ? sm + S_BS : sm + S_GN + cur * 16384;
                const uint4 v = *reinterpret_cast<const uint4*>(src + staged_off(row, ch));
                if (tile == 0) *reinterpret_cast<uint4*>(a.dx + grow * kP + 4 * ch) = v;
                else *reinterpret_cast<uint4*>((tile == 1 ? a.wdB : a.wdC) + grow * kN + 8 * ch) = v;
            }
        }
        fence_before_sync();
        __syncthreads();
        fence_after_sync();
        if (s_abort) break;
        if (tid == 0 && c > 0) issue_b(c - 1);   // theta copied, dY and Cbar read

        // ---- the angle adjoint's suffix sum over the sequence: dPhi_t = carry + sum_{s>=t} dl_s;
        // dtheta = dt dPhi; theta . dPhi per token (4 segments of Q / 4 tokens per pair) ----
        {
            constexpr int QS = Q / 4;
            const int i = tid & 63, sg = tid >> 6;
            // the segment's angle adjoints in registers first, so that the loads do not wait on
            // one another
            float dlv[QS];
            float loc = 0.f;
#pragma unroll
            for (int k = 0; k < QS; ++k) {
                dlv[k] = sphi[(QS * sg + k) * kPhiStride + i];
                loc += dlv[k];
            }
            s_suf[sg * 64 + i] = loc;
            __syncthreads();
            float acc = s_car[i];
            for (int s2 = 3; s2 > sg; --s2) acc += s_suf[s2 * 64 + i];
            float* dth = a.dtheta + ((bb * L + t0) * H + hh) * kHalf + i;
#pragma unroll
            for (int k = QS - 1; k >= 0; --k) {
                const int t = QS * sg + k;
                acc += dlv[k];
                float thd = 0.f;
                if (t < T) {
                    dth[static_cast<int64_t>(t) * H * kHalf] = sf[F_DT + t] * acc;
                    const uint16_t thb = *reinterpret_cast<const uint16_t*>(sm + S_PS + swz128(t, i));
                    thd = __uint_as_float(static_cast<uint32_t>(thb) << 16) * acc;
                }
                sphi[t * kPhiStride + i] = thd;
            }
            __syncthreads();
            if (sg == 0) s_car[i] += s_suf[i] + s_suf[64 + i] + s_suf[128 + i] + s_suf[192 + i];
            // row sums of theta . dPhi (4 threads per token), dy . y, out to the token's slots
            const int t = tid >> 2, qq = tid & 3;
            float s = 0.f;
#pragma unroll
            for (int k = 0; k < 16; ++k) s += sphi[t * kPhiStride + 16 * qq + k];
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (qq == 0 && t < T) a.wsc[(u * L + t0 + t) * 4 + 3] = s;
        }
        // ---- the decay gradient's per-token term (warp 0). D_t = <G_t, alpha_t h_{t-1}> =
        // D'_t - beta_t db_t with D'_t = T1 + T2 + T3 + T4:
        //   T1 = sum over pairs s' < t <= s of e^{cum_s - cum_s'} w_s' S'[s',s] Z[s',s]
        //        (a prefix over t of row sums minus column sums of the crossing entries),
        //   T2 = sum_{s >= t} e^{cum_s - cum_0} dy_s . Yo_s   (the chunk-start state),
        //   T3 = sum_{s' < t} w_s' e^{cx_T - cum_s'} q_s'     (the next chunk's adjoint),
        //   T4 = e^{cx_T - cum_0} <G_n, e^{cum_0} H0'>.
        // The sequential form's suffix sum over dy.y - beta db - gamma dg is replaced by these
        // per-chunk sums: its slot 2 receives D_t - D_{t+1} + beta_t db_t + gamma_t dg_t, so the
        // scalar kernel's suffix sum gives D_t without the cancellation of the long difference.
        if (warp == 0) {
            float g[2], p3[2], v[2];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                float ru = 0.f, q = 0.f, vv = 0.f, cu = 0.f;
                const bool real = t < T;
                if (real) {
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int row = t * R + r;
#pragma unroll
                        for (int s4 = 0; s4 < 4; ++s4) {
                            ru += red[(R_RU * 4 + s4) * 64 + row];
                            q += red[(R_Q * 4 + s4) * 64 + row];
                            vv += red[(R_V * 4 + s4) * 64 + row];
                            cu += s_cu[s4 * 64 + row];
                        }
                    }
                }
                g[k] = real ? ru - cu : 0.f;
                p3[k] = real ? sf[F_VN + t] * q : 0.f;
                v[k] = real ? sf[F_DS + t] * vv : 0.f;
            }
            // exclusive prefixes of g and p3, inclusive suffix of v, over the chunk's tokens (<= 64)
            const float gi0 = warp_inclusive_scan(g[0]), gi1 = warp_inclusive_scan(g[1]);
            const float pi0 = warp_inclusive_scan(p3[0]), pi1 = warp_inclusive_scan(p3[1]);
            const float vi0 = warp_inclusive_scan(v[0]), vi1 = warp_inclusive_scan(v[1]);
            const float gt0 = __shfl_sync(0xffffffffu, gi0, 31), pt0 = __shfl_sync(0xffffffffu, pi0, 31);
            const float vt0 = __shfl_sync(0xffffffffu, vi0, 31), vt1 = __shfl_sync(0xffffffffu, vi1, 31);
            float t4 = 0.f;
#pragma unroll
            for (int w8 = 0; w8 < 8; ++w8) t4 += s_t4[w8];
            t4 *= sf[F_MISC + 0];
            float dp[2];
            dp[0] = (gi0 - g[0]) + (vt0 + vt1 - vi0 + v[0]) + (pi0 - p3[0]) + t4;
            dp[1] = (gt0 + gi1 - g[1]) + (vt1 - vi1 + v[1]) + (pt0 + pi1 - p3[1]) + t4;
            const float dnext = s_dnext;
            const float dp1_0 = __shfl_down_sync(0xffffffffu, dp[0], 1);
            const float dp1_1 = __shfl_down_sync(0xffffffffu, dp[1], 1);
            const float dp_32 = __shfl_sync(0xffffffffu, dp[1], 0);
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = lane + 32 * k;
                if (t < T) {
                    const float db1 = s_tok[64 + t];
                    float dnx;   // D_{t+1}
                    if (t + 1 < T) {
                        const float dpn = k ? dp1_1 : (lane == 31 ? dp_32 : dp1_0);
                        dnx = dpn - sf[F_BETA + t + 1] * db1;
                    } else {
                        dnx = dnext - sf[F_BETA + Q] * db1;
                    }
                    // D'_t - D_{t+1} + gamma_t dg_t: the scalar kernel subtracts beta_t db_t and
                    // gamma_t dg_t again, leaving D_t - D_{t+1} (D_t = D'_t - beta_t db_t)
                    a.wsc[(u * L + t0 + t) * 4 + 2] = dp[k] - dnx + sf[F_GAM + t] * s_tok[t];
                }
            }
            __syncwarp();
            if (lane == 0) s_dnext = dp[0];
        }
        __syncthreads();
    }

    // ---------------- the initial state's gradients (token -1) ----------------
    if (!s_abort && nch > 0) {
        // chunk 0's scalars are still in place: alpha_0, beta_0
        const float al0 = sf[F_MISC + 1], be0 = sf[F_MISC + 2];
        if (a.dh0) {
            float4* dst = reinterpret_cast<float4*>(a.dh0 + (u * kN + nrow) * kP + 32 * wh);
#pragma unroll
            for (int j = 0; j < 8; ++j)
                dst[j] = make_float4(al0 * gr[4 * j], al0 * gr[4 * j + 1], al0 * gr[4 * j + 2], al0 * gr[4 * j + 3]);
        }
        // Bbar_{-1}[r] (the stored raw B, normalised, biased, rotated by phi0) and x_{-1}[r],
        // in buffers the loop no longer uses (no copy is in flight after chunk 0)
        float* w1 = reinterpret_cast<float*>(sm + S_CT);   // 8192 floats (raw C and raw B)
        float* pb = w1;                // [R][128] Bbar_{-1}
        float* px = w1 + 1024;         // [R][64]  x_{-1}
        float* pcs = w1 + 1536;        // [64] cos, [64] sin of phi0
        float* pred = w1 + 1664;       // [8] db_0 partials, [8 + r] the RMS scales
        float* pgx = w1 + 1696;        // [2][R][128] (G_0 x_{-1}[r]) halves, then dBbar_{-1}
        float* pdx = w1 + 3744;        // [4][R][64] dprevx partials
        float* pbias = w1 + 5792;      // [R][128] dBbar_{-1} rotated back, for the bias sum
        const __nv_bfloat16* pB = static_cast<const __nv_bfloat16*>(p.prevB0);
        if (warp < R) {
            float ss = 0.f;
            for (int n = lane; n < kN; n += 32) {
                const float v = pB ? __bfloat162float(pB[(u * R + warp) * kN + n]) : 0.f;
                ss += v * v;
            }
            ss = warp_sum(ss);
            if (lane == 0) pred[8 + warp] = p.bc_norm ? rsqrtf(ss / kN + p.eps) : 1.f;
        }
        __syncthreads();
        for (int e = tid; e < R * kHalf; e += kThreads) {
            const int r = e / kHalf, i = e % kHalf;
            const float rsp = pred[8 + r];
            const int64_t o = (u * R + r) * kN;
            const float u0 = (pB ? __bfloat162float(pB[o + i]) : 0.f) * rsp + s_bias[r * kN + i];
            const float u1 = (pB ? __bfloat162float(pB[o + i + kHalf]) : 0.f) * rsp + s_bias[r * kN + i + kHalf];
            float sn, cs;
            sincosf(p.phi0 ? p.phi0[u * kHalf + i] : 0.f, &sn, &cs);
            pb[r * kN + i] = u0 * cs + u1 * sn;
            pb[r * kN + i + kHalf] = u1 * cs - u0 * sn;
            if (r == 0) {
                pcs[i] = cs;
                pcs[kHalf + i] = sn;
            }
            px[e] = p.prevx0 ? __bfloat162float(static_cast<const __nv_bfloat16*>(p.prevx0)[u * R * kP + e]) : 0.f;
        }
        __syncthreads();
#pragma unroll 1
        for (int r = 0; r < R; ++r) {
            // (G_0 x_{-1}[r])[n] partial over this thread's columns; dprevx0 partials over rows
            float gx = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) gx = fmaf(gr[j], px[r * kP + 32 * wh + j], gx);
            pgx[(wh * R + r) * kN + nrow] = gx;
            const float bn = pb[r * kN + nrow];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const float v = warp_sum(bn * gr[j]);
                if (lane == j) pdx[(q4 * R + r) * kP + 32 * wh + j] = v;
            }
        }
        __syncthreads();
        {
            float v = 0.f;   // db_0 partial
            for (int e = tid; e < R * kN; e += kThreads) {
                const int r = e / kN, n = e % kN;
                const float gx = pgx[r * kN + n] + pgx[(R + r) * kN + n];
                v = fmaf(pb[e], gx, v);
                pgx[e] = be0 * gx;      // dBbar_{-1}[r][n]
            }
            v = warp_sum(v);
            if (lane == 0) pred[warp] = v;
        }
        __syncthreads();
        if (tid == 0) {
            float v = 0.f;
            for (int w = 0; w < kThreads / 32; ++w) v += pred[w];
            a.wsc[u * L * 4 + 0] = v;
        }
        if (a.dprevx0)
            for (int e = tid; e < R * kP; e += kThreads) {
                const int r = e / kP, pp = e % kP;
                float v = 0.f;
#pragma unroll
                for (int w4 = 0; w4 < 4; ++w4) v += pdx[(w4 * R + r) * kP + pp];
                a.dprevx0[u * R * kP + e] = be0 * v;
            }
        if (tid < kHalf) {
            const int i = tid;
            const float cs = pcs[i], sn = pcs[kHalf + i];
            float dl = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float d0 = pgx[r * kN + i], d1 = pgx[r * kN + i + kHalf];
                dl += d0 * pb[r * kN + i + kHalf] - d1 * pb[r * kN + i];
                const float n0 = d0 * cs - d1 * sn, n1 = d0 * sn + d1 * cs;
                a.wprev[(u * R + r) * kN + i] = n0;
                a.wprev[(u * R + r) * kN + i + kHalf] = n1;
                pbias[r * kN + i] = n0;
                pbias[r * kN + i + kHalf] = n1;
            }
            if (a.dphi0) a.dphi0[u * kHalf + i] = s_car[i] + dl;
        }
        __syncthreads();
        // bias sums: over the rows of one rank within each half-warp (its lanes differ in the
        // bits at and above R), then over the four row blocks, per rank
        float* sb = reinterpret_cast<float*>(sm + S_BT);   // [4][2][R][128]
        const int rk = trow % R;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            float vb = accB[k], vc = accC[k];
#pragma unroll
            for (int o = R; o < 16; o <<= 1) {
                vb += __shfl_xor_sync(0xffffffffu, vb, o);
                vc += __shfl_xor_sync(0xffffffffu, vc, o);
            }
            if ((lane & 15) < R) {
                const int col = col0 + (k & 15) + (k >= 16 ? kHalf : 0);
                sb[((q4 * 2 + 0) * R + rk) * kN + col] = vb;
                sb[((q4 * 2 + 1) * R + rk) * kN + col] = vc;
            }
        }
        __syncthreads();
        for (int e = tid; e < 2 * R * kN; e += kThreads) {
            const int isC = e / (R * kN), rem = e % (R * kN);
            float v = 0.f;
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) v += sb[(w4 * 2 + isC) * R * kN + rem];
            if (!isC) v += pbias[rem];
            a.wbias[u * 2 * R * kN + e] = v;
        }
    }

    if (s_abort && tid == 0) {
        if (a.status) atomicExch(a.status, 1);
        // let this CTA's own copies and MMAs finish (bounded) before TMEM is released
        constexpr long long kDrain = 200000000LL;
        if (s_lcnt[0] > 0) (void)mbar_wait(&bar_a, (s_lcnt[0] - 1) & 1, kDrain);
        if (s_lcnt[1] > 0) (void)mbar_wait(&bar_x, (s_lcnt[1] - 1) & 1, kDrain);
        if (s_lcnt[2] > 0) (void)mbar_wait(&bar_h, (s_lcnt[2] - 1) & 1, kDrain);
        if (s_lcnt[3] > 0) (void)mbar_wait(&bar_b, (s_lcnt[3] - 1) & 1, kDrain);
        if (s_cnt[1] > 0) (void)mbar_wait(&bar_m1, (s_cnt[1] - 1) & 1, kDrain);
        if (s_cnt[2] > 0) (void)mbar_wait(&bar_g, (s_cnt[2] - 1) & 1, kDrain);
        if (s_cnt[3] > 0) (void)mbar_wait(&bar_m2, (s_cnt[3] - 1) & 1, kDrain);
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// dB_bias[h] = sum over the batch of the units' sums (fixed order), and the same for C; RN is
// R * N, the bias length per head.
__global__ void __launch_bounds__(256) bwd_bias_sum_kernel(const float* __restrict__ wbias,
                                                           int64_t b, int64_t H, int RN,
                                                           float* dBbias, float* dCbias) {
    const int64_t h = blockIdx.x;
    for (int n = threadIdx.x; n < 2 * RN; n += blockDim.x) {
        float v = 0.f;
        for (int64_t i = 0; i < b; ++i) v += wbias[(i * H + h) * 2 * RN + n];
        if (n < RN) {
            if (dBbias) dBbias[h * RN + n] = v;
        } else if (dCbias) {
            dCbias[h * RN + n - RN] = v;
        }
    }
}

template <int R>
cudaError_t launch_bwd_tc_r(const BwdTcArgs& a, const BwdMaps& maps, int64_t units, bool raw,
                            cudaStream_t s) {
    auto kern = raw ? bwd_tc_kernel<R, true> : bwd_tc_kernel<R, false>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    kern<<<static_cast<unsigned>(units), kThreads, kSmemBytes, s>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace

bool bwd_tc_supported(const ScanParams& p, bool bf16) {
    if (p.R != 1 && p.R != 2 && p.R != 4 && p.R != 8) return false;
    ScanParams q = p;
    q.Q = kQ / p.R;
    return bf16 && tc_scan_supported(q, true);
}

size_t bwd_tc_workspace_bytes(const ScanParams& p) {
    const int64_t Q = kQ / p.R, nch = (p.L + Q - 1) / Q, units = p.b * p.H;
    auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
    return r256(static_cast<size_t>(units) * nch * 16384) +
           r256(static_cast<size_t>(units) * nch * kHalf * 4) +
           r256(static_cast<size_t>(units) * kN * kP * 4) +
           r256(static_cast<size_t>(units) * (kHalf + 1) * 4) +
           r256(static_cast<size_t>(units) * 2 * p.R * kN * 4) +
           r256(static_cast<size_t>(p.b) * nch * Q * p.G * p.R * sizeof(float2));
}

cudaError_t launch_bwd_tc(const ScanParams& p, const BwdTcOut& o, void* ws, cudaStream_t s) {
    const int64_t R = p.R, Q = kQ / R, nch = (p.L + Q - 1) / Q, units = p.b * p.H;
    auto r256 = [](size_t v) { return (v + 255) / 256 * 256; };
    uint8_t* w = static_cast<uint8_t*>(ws);
    BwdTcArgs a{};
    a.p = p;
    a.nch = static_cast<int>(nch);
    uint8_t* chunk_h = w; w += r256(static_cast<size_t>(units) * nch * 16384);
    float* chunk_phi = reinterpret_cast<float*>(w); w += r256(static_cast<size_t>(units) * nch * kHalf * 4);
    float* hfin = reinterpret_cast<float*>(w); w += r256(static_cast<size_t>(units) * kN * kP * 4);
    float* phifin = reinterpret_cast<float*>(w);
    float* lamfin = phifin + units * kHalf;
    w += r256(static_cast<size_t>(units) * (kHalf + 1) * 4);
    float* wbias = reinterpret_cast<float*>(w); w += r256(static_cast<size_t>(units) * 2 * R * kN * 4);
    float2* rs = p.bc_norm ? reinterpret_cast<float2*>(w) : nullptr;

    // the forward state pass: e^{cum_0} H0' and the angle before every chunk, the final state
    cudaError_t e = launch_bwd_states_tc(p, rs, chunk_h, chunk_phi, hfin, phifin, lamfin, s);
    if (e != cudaSuccess) return e;

    BwdMaps maps;
    const uint64_t H = p.H, Lq = p.L, b = p.b, G = p.G, Ru = static_cast<uint64_t>(R);
    const uint32_t Qb = static_cast<uint32_t>(Q), Rb = static_cast<uint32_t>(R);
    {   // x, dy [b][L][H][R][P], box (P, R, 1, Q, 1)
        const uint64_t dims[5] = {kP, Ru, H, Lq, b};
        const uint64_t str[4] = {kP * 2, Ru * kP * 2, H * Ru * kP * 2, Lq * H * Ru * kP * 2};
        const uint32_t box[5] = {kP, Rb, 1, Qb, 1};
        if (!encode_tmap(&maps.x, true, 5, p.x, dims, str, box, true) ||
            !encode_tmap(&maps.dy, true, 5, o.dy, dims, str, box, true))
            return cudaErrorInvalidValue;
    }
    {   // theta [b][L][H][N/2], box (64, 1, Q, 1)
        const uint64_t dims[4] = {kHalf, H, Lq, b};
        const uint64_t str[3] = {kHalf * 2, H * kHalf * 2, Lq * H * kHalf * 2};
        const uint32_t box[4] = {kHalf, 1, Qb, 1};
        if (!encode_tmap(&maps.theta, true, 4, p.theta, dims, str, box, true))
            return cudaErrorInvalidValue;
    }
    {   // B, C [b][L][G][R][N], box (64 columns, R, 1, Q, 1)
        const uint64_t dims[5] = {kN, Ru, G, Lq, b};
        const uint64_t str[4] = {kN * 2, Ru * kN * 2, G * Ru * kN * 2, Lq * G * Ru * kN * 2};
        const uint32_t box[5] = {kHalf, Rb, 1, Qb, 1};
        if (!encode_tmap(&maps.B, true, 5, p.B, dims, str, box, true) ||
            !encode_tmap(&maps.C, true, 5, p.C, dims, str, box, true))
            return cudaErrorInvalidValue;
    }
    {   // dt, A, lam [b][L][H] fp32, box (4 heads, Q + 1 tokens, 1)
        const uint64_t dims[3] = {H, Lq, b};
        const uint64_t str[2] = {H * 4, Lq * H * 4};
        const uint32_t box[3] = {4, Qb + 1, 1};
        if (!encode_tmap(&maps.dt, false, 3, p.dt, dims, str, box, false) ||
            !encode_tmap(&maps.A, false, 3, p.A, dims, str, box, false) ||
            !encode_tmap(&maps.lam, false, 3, p.lam, dims, str, box, false))
            return cudaErrorInvalidValue;
    }
    a.rs = rs;
    a.chunk_h = chunk_h;
    a.chunk_phi = chunk_phi;
    a.hfin = hfin;
    a.dh1 = o.dh1;
    a.dphi1 = o.dphi1;
    a.dprevx1 = o.dprevx1;
    a.dx = o.dx;
    a.dtheta = o.dtheta;
    a.wdB = static_cast<__nv_bfloat16*>(o.wdB);
    a.wdC = static_cast<__nv_bfloat16*>(o.wdC);
    a.wsc = o.wsc;
    a.wprev = o.wprev;
    a.wF = o.wF;
    a.wbias = wbias;
    a.dh0 = o.dh0;
    a.dphi0 = o.dphi0;
    a.dprevx0 = o.dprevx0;
    a.status = o.status;
    // test hook of the timeout path (as for the forward scans): > 0 makes CTA 0 skip the
    // theta / dY / raw C load of that step, so that its bounded wait gives up
    if (const char* env = std::getenv("M3_TEST_SKIP_THETA_LOAD")) a.p.test_skip_theta = std::atoi(env);
    const bool raw = p.flags != 0;
    switch (R) {
        case 1: e = launch_bwd_tc_r<1>(a, maps, units, raw, s); break;
        case 2: e = launch_bwd_tc_r<2>(a, maps, units, raw, s); break;
        case 4: e = launch_bwd_tc_r<4>(a, maps, units, raw, s); break;
        case 8: e = launch_bwd_tc_r<8>(a, maps, units, raw, s); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    if (o.dBbias || o.dCbias) {
        bwd_bias_sum_kernel<<<static_cast<unsigned>(p.H), 256, 0, s>>>(
            wbias, p.b, p.H, static_cast<int>(R * kN), o.dBbias, o.dCbias);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace m3
