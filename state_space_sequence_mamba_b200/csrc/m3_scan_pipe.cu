// Chunked prefill scan on the sm_100a tensor cores, warp-specialised, one CTA per SM.
//
// Method ("Mamba-3: Improved Sequence Modeling using State Space Principles", Sec. 3.1.3 eq. 7
// for the masked parallel form, Sec. 3.3 for the chunked algorithm and MIMO, Appendix B.3 for
// the rotated frame). The state carried between chunks is the primed state
//     h'_t = h~_t + (1 - lam_{t+1}) dt_{t+1} v_t,   v_t = sum_r Bbar_t[r] x_t[r]^T,
// which obeys h'_t = alpha_t h'_{t-1} + w_t v_t with w_t = gamma_t + (1 - lam_{t+1}) dt_{t+1}
// (w = gamma for the sequence's last token). A chunk is 128 rows: Q = 128 / R tokens of R
// (token, rank) rows each. With cum = the chunk-local inclusive sum of dt*A and ref = the
// midpoint of cum over the chunk, the decay mask of eq. 7 is moved into the operands: row s of
// Bbar is scaled by e^{ref - cum_s} w_s and row t of Cbar by e^{cum_t - ref} (both folded into
// the rotation's cos and sin), so that S' = Cbar' Bbar'^T is S o M below the diagonal,
// M[t,s] = e^{cum_t - cum_s} w_s (s < t), gamma_t (s = t), 0 (s > t). Per chunk:
//     S'  = Cbar' Bbar'^T                  M128 N128 K128 (A, B in shared memory)
//     dH' = Bbar'^T X                      M128 N64 K128
//     Y   = Cbar' (e^{ref} H0)             M128 N64 K128
//     P   = S' (s < t), S' gamma_t / w_t (s = t), 0 (s > t)   (TMEM -> registers -> TMEM, bf16)
//     Y  += P X                            M128 N64 K128 (A = P in TMEM); y = Y
//     H1  = e^{cum_end} H0 + e^{cum_end - ref} dH'
// Every factor stays within e^{+-30} while the chunk decays by at most 60 nats. A chunk that
// decays faster (strong decay) is computed exactly as written above instead: unit scales,
// dH from X' = diag(e^{cum_end - cum} w) X, the mask element by element and Y = Cbar H0
// rescaled row by row by e^{cum_t} before P X is added. MIMO rows are (token, rank) pairs; the
// token mask covers full R x R blocks.
//
// Roles (24 warps, 768 threads; every TMEM accumulator is 128 lanes, so TMEM reads use whole
// warps):
//   warps 8-23  rotation: the chunk's cumulative angles (each thread walks 4 rotation pairs
//               over a segment of tokens; segment offsets by a warp scan and per-warp totals),
//               B and C normalised, biased, rotated and scaled in place in their TMA stage in
//               fp32 with one rounding to bf16 (and X' in the exact mode). They work one
//               chunk ahead of the tensor cores: raw B, C, X and theta are double-buffered.
//   warps 0-3   TMEM: the state pass (state columns, the next H0 operand), the mask P
//               written back to TMEM as bf16, the epilogue y (one accumulator, double-buffered).
//   warp 4      one lane issues S', Yo and dH of every chunk (and their commit).
//   warp 5      one lane issues Yd = P X of every chunk (and its commit).
//   warp 6      one lane issues the TMA loads.
//   warp 7      the chunk scalars (cumulative decay, reference, operand factors, mode).
// Hand-offs are mbarriers (TMA transaction counts, tcgen05.commit, per-warp arrivals); in the
// rotation and TMEM groups one leader thread waits and a named barrier releases the group. All
// waits are bounded, and a wait that gives up records the status word and lets every role
// leave its loop.
#include <cstdlib>

#include <cuda.h>
#include <cudaTypedefs.h>

#include "m3_common.cuh"
#include "m3_internal.h"
#include "m3_sm100.cuh"

namespace m3 {

namespace {

using namespace sm100;

constexpr int kN = 128, kP = 64, kHalf = 64, kRows = 128;
// Warp order: the TMEM warps first (their chain gates every chunk, and the schedulers favour
// older warps), then the single-lane issuers and the scalar warp, then the rotation warps.
constexpr int kRWarps = 16, kTWarps = 4;
constexpr int kTWarp0 = 0;
constexpr int kMmaWarp = kTWarps;
constexpr int kYdWarp = kMmaWarp + 1;
constexpr int kLoadWarp = kYdWarp + 1;
constexpr int kScalWarp = kLoadWarp + 1;
constexpr int kRWarp0 = kScalWarp + 1;
constexpr int kThreads = (kRWarp0 + kRWarps) * 32;
constexpr int kRThreads = kRWarps * 32;

// TMEM columns: S' x2 (fp32, 128 each), P (bf16 pairs, 64), the state H (64), Y x2 (64 each).
// The state columns hold sigma H(c) before chunk c's dH MMA accumulates onto them (sigma =
// e^{ref}, or e^{cum_end} in the exact mode), so that afterwards they hold H(c+1) / xs with
// xs = e^{cum_end - ref} (1 in the exact mode).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t T_S = 0, T_P = 256, T_H = 320, T_Y = 384;

// One chunk's scalars (floats), three blocks in turn (chunk c in block c % 3), per token: dt;
// A1, A2 = the Bbar and Cbar row factors (scaled mode) or log2-scaled cum and w (exact mode);
// gamma / w (scaled mode) or gamma (exact mode). MISC: e^{cum_end}, the mode (0 scaled,
// 1 exact), the dH' factor xs = e^{cum_end - ref}, the H0 factor e^{ref} (1, 1 in the exact
// mode), log2-scaled cum_end.
constexpr int kScBufs = 3;
constexpr int SC_DT = 0, SC_A1 = 128, SC_A2 = 256, SC_GW = 384, SC_MISC = 512, SC_FLOATS = 528;
constexpr int MISC_EEND = 0, MISC_MODE = 1, MISC_XS = 2, MISC_EH0 = 3, MISC_CEND2 = 4;
// sigma of the state columns before a chunk's dH MMA: e^{ref}, or e^{cum_end} in the exact mode
__device__ __forceinline__ float state_sigma(const float* sc) {
    return sc[SC_MISC + MISC_MODE] != 0.f ? sc[SC_MISC + MISC_EEND] : sc[SC_MISC + MISC_EH0];
}
// the largest chunk decay (nats) the scaled mode takes: every factor <= e^30
constexpr float kMaxChunkDecay = 60.f;

// mbarriers (pairs and triples: one per buffer)
enum {
    B_TH_FULL, B_TH_FULL1, B_TH_EMPTY, B_TH_EMPTY1, B_BC_FULL, B_BC_FULL1, B_BC_EMPTY, B_BC_EMPTY1,
    B_X_FULL, B_X_FULL1, B_X_EMPTY, B_X_EMPTY1, B_SC_READY, B_SC_READY1, B_SC_READY2, B_SC_FREE,
    B_SC_FREE1, B_SC_FREE2, B_OPS, B_OPS1, B_XP_EMPTY, B_XP_EMPTY1, B_S_FREE, B_S_FREE1, B_DH_FREE,
    B_SD_FULL, B_H0_FULL, B_Y_FREE, B_Y_FREE1, B_P_FULL, B_YD_FULL, B_DRAIN, B_DRAIN2, kNumBars
};
__host__ __device__ constexpr uint32_t bar_count(int b) {
    return (b == B_TH_EMPTY || b == B_TH_EMPTY1 || b == B_OPS || b == B_OPS1) ? kRWarps
         : (b >= B_SC_FREE && b <= B_SC_FREE2) ? kRWarps + kTWarps
         : (b == B_S_FREE || b == B_S_FREE1 || b == B_DH_FREE || b == B_H0_FULL || b == B_Y_FREE || b == B_Y_FREE1 ||
            b == B_P_FULL) ? kTWarps
         : 1;
}

template <int R>
struct PCfg {
    static constexpr int Q = kRows / R;          // tokens per chunk
    static constexpr int TPS = Q / 32;           // tokens per rotation segment (32 segments)
    static constexpr int TPL = Q / 32;           // tokens per lane of the scalar warp
    static_assert(TPS >= 1, "ranks 1, 2, 4");
    // shared-memory byte layout after 1024-byte alignment
    static constexpr uint32_t SLAB = 16384;      // 64 columns of a 128-row swizzled operand
    static constexpr uint32_t BC_STAGE = 65536;  // [Bbar slab 0, slab 1, Cbar slab 0, slab 1]
    static constexpr uint32_t C_OFF = 32768;
    static constexpr uint32_t X0 = 131072, X_STAGE = 16384;   // X, two stages (TMA)
    static constexpr uint32_t TH0 = 163840, TH_STAGE = Q * 128;  // theta, two stages (TMA)
    // X' = diag(dw) X (exact mode): in the chunk's own theta stage when that holds 128 rows
    // (R = 1), else in a buffer of its own
    static constexpr uint32_t XP = TH0 + 2 * TH_STAGE;
    static constexpr uint32_t XP_BYTES = (R == 1) ? 0 : 16384;
    static constexpr uint32_t H0 = XP + XP_BYTES;             // H0 bf16 [n][p]
    static constexpr uint32_t RS = H0 + 16384;                // RMS scales [2][128] float2
    static constexpr uint32_t SC = RS + 2 * kRows * 8;        // scalars [3][SC_FLOATS]
    static constexpr uint32_t BIAS = SC + kScBufs * SC_FLOATS * 4;  // bias [B, C][R][2][16][4]
    static constexpr uint32_t WT = BIAS + 2 * R * kN * 4;     // warp angle totals [16][64]
    static constexpr uint32_t PHI = WT + kRWarps * kHalf * 4; // unreduced angle [64]
    static constexpr uint32_t CARRY = PHI + kHalf * 4;        // reduced angle carry [2][64]
    static constexpr uint32_t END = CARRY + 2 * kHalf * 4;
    static constexpr uint32_t SMEM = END + 1024;
    static constexpr uint32_t BC_TX = 4 * SLAB;               // raw B and raw C
    static constexpr uint32_t X_TX = 16384;
    static constexpr uint32_t TH_TX = Q * 128;
    __host__ __device__ static constexpr uint32_t xp(int st) {
        return R == 1 ? TH0 + static_cast<uint32_t>(st) * TH_STAGE : XP;
    }
};
static_assert(PCfg<1>::SMEM + 512 <= 232448, "shared memory (R = 1)");
static_assert(PCfg<2>::SMEM + 512 <= 232448, "shared memory (R = 2)");
static_assert(PCfg<4>::SMEM + 512 <= 232448, "shared memory (R = 4)");

// 2^x by the hardware approximation (relative error ~2^-22), x <= 0 here.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two floats rounded to bf16 and packed (a in the low half).
__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint32_t pack2(float2 v) { return pack_bf16(v.x, v.y); }
// The same on the integer pipe, for the rotation warps (whose sine and cosine keep the
// conversion pipe busy): half an ulp of bf16 is added to the bit pattern and the high halves
// are kept, which rounds to nearest with ties away from zero (finite inputs).
__device__ __forceinline__ uint32_t pack2_alu(float2 v) {
    return __byte_perm(__float_as_uint(v.x) + 0x8000u, __float_as_uint(v.y) + 0x8000u, 0x7632);
}
// (low, high) bf16 halves of a word as exact fp32
__device__ __forceinline__ float2 unpack2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

struct PMaps {
    CUtensorMap x, theta, B, C;
};

// Waits for the phase of `bar` with the given parity, giving up when another role has
// recorded an abort or after ~max_cycles SM clocks (then records the abort itself). Between
// checks the warp is suspended in the wait instruction itself (up to kSuspendNs, or until the
// phase completes), so waiting roles take no issue slots from the working ones.
constexpr uint32_t kSuspendNs = 100000;
__device__ __forceinline__ bool pwait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                      long long max_cycles = 2000000000LL) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait_sleep(a, parity & 1u, kSuspendNs)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(a, parity & 1u, kSuspendNs)) return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > max_cycles) {
            *abort_flag = 1;
            return false;
        }
    }
}

template <int R, bool kRaw>
__global__ void __launch_bounds__(kThreads, 1)
scan_pipe_kernel(const ScanParams p, const __grid_constant__ PMaps maps,
                 const float2* __restrict__ rsrow) {
    using Cfg = PCfg<R>;
    constexpr int Q = Cfg::Q, TPS = Cfg::TPS, TPL = Cfg::TPL;

    // the operand tiles want 1024-byte alignment; offsetting the shared array itself (not a
    // generic pointer) keeps every access below a shared-memory access
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    __shared__ __align__(8) uint64_t bars[kNumBars];
    __shared__ uint32_t tslot;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t u = blockIdx.x;
    const int64_t bb = u / p.H, hh = u % p.H, g = hh / (p.H / p.G);
    const int L = static_cast<int>(p.L), H = static_cast<int>(p.H), G = static_cast<int>(p.G);
    const int nchunks = (L + Q - 1) / Q;
    const int Lpad = nchunks * Q;
    const int ib = static_cast<int>(bb), ih = static_cast<int>(hh), ig = static_cast<int>(g);
    const float2* rsu = rsrow ? rsrow + (bb * G + g) * static_cast<int64_t>(Lpad) * R : nullptr;
    // Per-unit base pointers; offsets below fit in 32 bits (checked on the host).
    const __nv_bfloat16* Bu = static_cast<const __nv_bfloat16*>(p.B) + (bb * p.L * G + g) * R * kN;
    const __nv_bfloat16* xu = static_cast<const __nv_bfloat16*>(p.x) + (bb * p.L * H + hh) * R * kP;
    __nv_bfloat16* yu = static_cast<__nv_bfloat16*>(p.y) + (bb * p.L * H + hh) * R * kP;
    const int tokB = G * R * kN, tokY = H * R * kP;   // element stride of one token
    float* s_sc = reinterpret_cast<float*>(sm + Cfg::SC);        // [3][SC_FLOATS]
    float* s_bias = reinterpret_cast<float*>(sm + Cfg::BIAS);    // [B, C][R][2][16][4]
    float* s_wt = reinterpret_cast<float*>(sm + Cfg::WT);        // [16 warps][64]
    float* s_phi = reinterpret_cast<float*>(sm + Cfg::PHI);      // unreduced angle [64]
    float* s_carry = reinterpret_cast<float*>(sm + Cfg::CARRY);  // [2][64]
    const float dtb = (kRaw && p.dt_bias) ? p.dt_bias[hh] : 0.f;   // only with M3_DT_SOFTPLUS

    // ---------------- set-up ----------------
    if (tid == 0) {
        for (int i = 0; i < kNumBars; ++i) mbar_init(&bars[i], bar_count(i));
        fence_mbar_init();
        s_abort = 0;
    }
    if (warp == 0) tmem_alloc(&tslot, kTmemCols);
    // biases, laid out so that the sixteen 4-pair blocks of one half are contiguous: element
    // ((tensor * R + r) * 2 + h) * 64 + 4 j + e holds n = 4 j + e + 64 h
    for (int i = tid; i < 2 * R * kN; i += kThreads) {
        const int e = i & 3, jj = (i >> 2) & 15, hf = (i >> 6) & 1, tr = i >> 7;   // tr = tensor * R + r
        const int tc = tr / R, r = tr % R;
        const float* src = tc ? p.Cbias : p.Bbias;
        s_bias[i] = src ? src[(hh * R + r) * kN + 4 * jj + e + 64 * hf] : 0.f;
    }
    if (tid < kHalf) {   // the carried angle: reduced for the walk, unreduced for the output
        const float ph0 = p.phi0 ? p.phi0[u * kHalf + tid] : 0.f;
        s_carry[tid] = reduce_2pi(ph0);
        s_phi[tid] = ph0;
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = tslot;

    // The stored previous token folded into the primed initial state (its beta term belongs to
    // this call's first token): Bbar_prev = R(-phi0)(norm(B_prev) + bias), weight
    // (1 - lam_0) dt_0. Scratch in the first theta stage, set-up only (its first load is
    // issued after set-up).
    float* s_fold = reinterpret_cast<float*>(sm + Cfg::TH0);   // [R][128]
    float* s_foldx = s_fold + R * kN;                           // [R][64]
    float* s_foldrs = s_foldx + R * kP;                         // [R]
    const bool fold = p.h0 && L > 0;
    float fold_w = 0.f;
    if (fold) {
        const __nv_bfloat16* pB = static_cast<const __nv_bfloat16*>(p.prevB0) + u * R * kN;
        const __nv_bfloat16* px = static_cast<const __nv_bfloat16*>(p.prevx0) + u * R * kP;
        if (warp < R) {
            float ss = 0.f;
            for (int n = lane; n < kN; n += 32) {
                const float v = __bfloat162float(pB[warp * kN + n]);
                ss = fmaf(v, v, ss);
            }
            ss = warp_sum(ss);
            if (lane == 0) s_foldrs[warp] = p.bc_norm ? rsqrtf(ss / kN + p.eps) : 1.f;
        }
        for (int i = tid; i < R * kP; i += kThreads) s_foldx[i] = __bfloat162float(px[i]);
        __syncthreads();
        for (int k = tid; k < R * kHalf; k += kThreads) {
            const int r = k / kHalf, i = k % kHalf;
            float sn, cs;
            sincosf(p.phi0[u * kHalf + i], &sn, &cs);
            const float rs = s_foldrs[r];
            const float b0 = p.Bbias ? p.Bbias[(hh * R + r) * kN + i] : 0.f;
            const float b1 = p.Bbias ? p.Bbias[(hh * R + r) * kN + i + kHalf] : 0.f;
            const float u0 = fmaf(__bfloat162float(pB[r * kN + i]), rs, b0);
            const float u1 = fmaf(__bfloat162float(pB[r * kN + i + kHalf]), rs, b1);
            s_fold[r * kN + i] = u0 * cs + u1 * sn;
            s_fold[r * kN + i + kHalf] = u1 * cs - u0 * sn;
        }
        const int64_t s0 = bb * p.L * p.H + hh;
        fold_w = (kRaw && (p.flags & 4u)) ? 0.f   // zero-order hold: no beta term
                 : (1.f - step_lam<kRaw>(p.lam[s0], p.flags)) * step_dt<kRaw>(p.dt[s0], dtb, p.flags);
        __syncthreads();
    }

    // TMEM warps: the initial state row n = 32 q + lane (with the folded token) into the state
    // columns, unscaled; the TMEM warps scale it once the first chunk's scalars are known
    const int tq = warp - kTWarp0;                 // TMEM subpartition of a TMEM warp
    const int nrow = 32 * tq + lane;
    const uint32_t lanebase = (32u * (warp & 3)) << 16;
    if (warp >= kTWarp0 && warp < kMmaWarp) {
        float bq[R];
#pragma unroll
        for (int r = 0; r < R; ++r) bq[r] = fold ? fold_w * s_fold[r * kN + nrow] : 0.f;
#pragma unroll
        for (int q16 = 0; q16 < 4; ++q16) {
            float hv[16];
            if (p.h0) {
                const float4* src = reinterpret_cast<const float4*>(p.h0 + (u * kN + nrow) * kP + 16 * q16);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float4 v = src[i];
                    hv[4 * i] = v.x; hv[4 * i + 1] = v.y; hv[4 * i + 2] = v.z; hv[4 * i + 3] = v.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) hv[i] = 0.f;
            }
            if (fold) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
#pragma unroll
                    for (int r = 0; r < R; ++r) hv[i] = fmaf(bq[r], s_foldx[r * kP + 16 * q16 + i], hv[i]);
            }
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(hv[i]);
            tmem_st_32x32b_x16(tmem + lanebase + T_H + 16u * q16, w);
        }
        tmem_wait_st();
    }
    fence_before_sync();
    __syncthreads();   // the fold scratch (first theta stage) has been read
    fence_after_sync();
    // One pass over the state columns after chunk c's dH (or, c = -1, over the initial state):
    // h = xs * columns is the state before the next chunk; it goes back times that chunk's
    // sigma and, times its H0 factor, to the H0 operand (or, after the last chunk, to the
    // caller's final state).
    auto state_pass = [&](float xs, const float* scn, bool last) {
        const float2 xs2 = make_float2(xs, xs);
        const float sg = last ? 1.f : state_sigma(scn);
        const float eh = last ? 1.f : scn[SC_MISC + MISC_EH0];
        const float2 sg2 = make_float2(sg, sg), eh2 = make_float2(eh, eh);
        const bool same = sg == eh;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
            float v[32];
            tmem_ld_32x32b_x32(tmem + lanebase + T_H + 32u * hf, v);
            tmem_wait_ld();
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int q16 = 2 * hf + q;
                float2 h[8];
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    h[i] = __fmul2_rn(xs2, make_float2(v[16 * q + 2 * i], v[16 * q + 2 * i + 1]));
                if (last) {
                    if (p.h1) {
                        float4* dst = reinterpret_cast<float4*>(p.h1 + (u * kN + nrow) * kP + 16 * q16);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dst[i] = make_float4(h[2 * i].x, h[2 * i].y, h[2 * i + 1].x, h[2 * i + 1].y);
                    }
                } else {
                    uint32_t w[16], hb[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float2 a = __fmul2_rn(sg2, h[i]);
                        w[2 * i] = __float_as_uint(a.x);
                        w[2 * i + 1] = __float_as_uint(a.y);
                        hb[i] = pack2(same ? a : __fmul2_rn(eh2, h[i]));   // scaled mode: sigma = e^{ref}
                    }
                    tmem_st_32x32b_x16(tmem + lanebase + T_H + 16u * q16, w);
                    *reinterpret_cast<uint4*>(sm + Cfg::H0 + swz128(nrow, 16 * q16)) = make_uint4(hb[0], hb[1], hb[2], hb[3]);
                    *reinterpret_cast<uint4*>(sm + Cfg::H0 + swz128(nrow, 16 * q16 + 8)) = make_uint4(hb[4], hb[5], hb[6], hb[7]);
                }
            }
        }
        if (!last) {
            tmem_wait_st();
            fence_proxy_async();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_DH_FREE]);
                mbar_arrive(&bars[B_H0_FULL]);
            }
        }
    };

    if (warp >= kRWarp0) {
        // ================= rotation warps =================
        // Thread = (segment sidx of TPS consecutive tokens, pair block j): rotation pairs
        // (i, i + N/2) for i in [4 j, 4 j + 4), an 8-byte piece of a 128-byte operand row.
        const int rw = warp - kRWarp0;   // rotation warp index
        const int j = lane & 15, sl = lane >> 4, sidx = rw * 2 + sl;
        const bool last_seg = (sidx == 31);
        auto piece = [&](int row) -> uint32_t {   // byte offset of this thread's piece of a row
            return static_cast<uint32_t>(row) * 128u +
                   (static_cast<uint32_t>(((j >> 1) ^ row) & 7) << 4) + (static_cast<uint32_t>(j & 1) << 3);
        };
        // the thread's rows are 4 sidx + i (i < 4: TPS tokens of R rows) and its theta rows
        // sidx TPS + k: their offsets once
        uint32_t roff[4], toff[TPS];
#pragma unroll
        for (int i = 0; i < 4; ++i) roff[i] = piece(4 * sidx + i);
#pragma unroll
        for (int k = 0; k < TPS; ++k) toff[k] = piece(sidx * TPS + k);
        const bool lead = (rw == 0 && lane == 0);   // waits for the group
        for (int c = 0; c < nchunks; ++c) {
            const int st = c & 1;
            const int sb3 = c % kScBufs;
            const float* sc = s_sc + sb3 * SC_FLOATS;
            bool fail = false;
            if (lead) fail = !pwait(&bars[B_SC_READY + sb3], c / kScBufs, &s_abort) ||
                             !pwait(&bars[B_TH_FULL + st], c >> 1, &s_abort);
            if (bar_sync_or(1, kRThreads, fail || s_abort)) break;   // scalars and theta are here
            const uint8_t* th = sm + Cfg::TH0 + st * Cfg::TH_STAGE;
            // the sum of this segment's angle increments dt_t theta_t
            float seg[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int k = 0; k < TPS; ++k) {
                const int t = sidx * TPS + k;
                const float d = sc[SC_DT + t];   // 0 past the sequence end: no rotation there
                const uint2 tw = *reinterpret_cast<const uint2*>(th + toff[k]);
                const float2 f0 = unpack2(tw.x), f1 = unpack2(tw.y);
                seg[0] = fmaf(d, f0.x, seg[0]); seg[1] = fmaf(d, f0.y, seg[1]);
                seg[2] = fmaf(d, f1.x, seg[2]); seg[3] = fmaf(d, f1.y, seg[3]);
            }
            // the warp's two segments (lanes j and j + 16), then the warps' totals
            float incl[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float o = __shfl_up_sync(0xffffffffu, seg[i], 16);
                incl[i] = sl ? seg[i] + o : seg[i];
            }
            if (sl == 1)
                *reinterpret_cast<float4*>(s_wt + rw * kHalf + 4 * j) = make_float4(incl[0], incl[1], incl[2], incl[3]);
            if (bar_sync_or(1, kRThreads, s_abort)) break;
            // angle before this segment: carry + earlier warps' totals + the earlier segment here
            const float4 cin = *reinterpret_cast<const float4*>(s_carry + st * kHalf + 4 * j);
            float a[4] = {cin.x, cin.y, cin.z, cin.w};
            for (int w = 0; w < rw; ++w) {
                const float4 t4 = *reinterpret_cast<const float4*>(s_wt + w * kHalf + 4 * j);
                a[0] += t4.x; a[1] += t4.y; a[2] += t4.z; a[3] += t4.w;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) a[i] += incl[i] - seg[i];
            if (last_seg) {   // the chunk-end angle: next chunk's carry (reduced) and the true sum
                const float cinv[4] = {cin.x, cin.y, cin.z, cin.w};
                float e[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    e[i] = a[i] + seg[i];
                    s_phi[4 * j + i] += e[i] - cinv[i];   // only this thread touches these
                    e[i] = reduce_2pi(e[i]);
                }
                *reinterpret_cast<float4*>(s_carry + (st ^ 1) * kHalf + 4 * j) = make_float4(e[0], e[1], e[2], e[3]);
            }
            if (lead) fail = !pwait(&bars[B_BC_FULL + st], c >> 1, &s_abort);   // raw B, C, RMS scales
            if (bar_sync_or(1, kRThreads, fail || s_abort)) break;   // and the warp totals have been read
            const bool exact = sc[SC_MISC + MISC_MODE] != 0.f;
            const bool norm = p.bc_norm != 0;
            uint8_t* sB = sm + st * Cfg::BC_STAGE;
            const float2* srs = reinterpret_cast<const float2*>(sm + Cfg::RS + st * (kRows * 8));
#pragma unroll
            for (int k = 0; k < TPS; ++k) {
                const int t = sidx * TPS + k;
                const float d = sc[SC_DT + t];
                {
                    const uint2 tw = *reinterpret_cast<const uint2*>(th + toff[k]);
                    const float2 f0 = unpack2(tw.x), f1 = unpack2(tw.y);
                    a[0] = fmaf(d, f0.x, a[0]); a[1] = fmaf(d, f0.y, a[1]);
                    a[2] = fmaf(d, f1.x, a[2]); a[3] = fmaf(d, f1.y, a[3]);
                }
                float2 cs01, cs23, sn01, sn23;
                __sincosf(a[0], &sn01.x, &cs01.x);
                __sincosf(a[1], &sn01.y, &cs01.y);
                __sincosf(a[2], &sn23.x, &cs23.x);
                __sincosf(a[3], &sn23.y, &cs23.y);
                // cos and sin times the token's B and C row factors (1 in the exact mode)
                const float fb = exact ? 1.f : sc[SC_A1 + t], fc = exact ? 1.f : sc[SC_A2 + t];
#pragma unroll
                for (int tc = 0; tc < 2; ++tc) {   // B, then C
                    const float f = tc ? fc : fb;
                    const float2 f2 = make_float2(f, f);
                    const float2 c0 = __fmul2_rn(cs01, f2), c1 = __fmul2_rn(cs23, f2);
                    const float2 s0 = __fmul2_rn(sn01, f2), s1 = __fmul2_rn(sn23, f2);
                    uint8_t* base = sB + tc * Cfg::C_OFF;
                    const float* bias = s_bias + tc * R * kN + 4 * j;
#pragma unroll
                    for (int r = 0; r < R; ++r) {
                        const int row = t * R + r;   // = 4 sidx + k R + r
                        const uint32_t o = roff[k * R + r];
                        const float rv = norm ? (tc ? srs[row].y : srs[row].x) : 1.f;
                        const float2 rv2 = make_float2(rv, rv);
                        const float4 b0 = *reinterpret_cast<const float4*>(bias + r * kN);
                        const float4 b1 = *reinterpret_cast<const float4*>(bias + r * kN + 64);
                        const uint2 w0 = *reinterpret_cast<const uint2*>(base + o);
                        const uint2 w1 = *reinterpret_cast<const uint2*>(base + Cfg::SLAB + o);
                        // u = rs * raw + bias on both halves of the pair, then
                        // (u0, u1) -> f (u0 cos + u1 sin, u1 cos - u0 sin)
                        const float2 u00 = __ffma2_rn(unpack2(w0.x), rv2, make_float2(b0.x, b0.y));
                        const float2 u01 = __ffma2_rn(unpack2(w0.y), rv2, make_float2(b0.z, b0.w));
                        const float2 u10 = __ffma2_rn(unpack2(w1.x), rv2, make_float2(b1.x, b1.y));
                        const float2 u11 = __ffma2_rn(unpack2(w1.y), rv2, make_float2(b1.z, b1.w));
                        const float2 t00 = __fmul2_rn(u00, s0), t01 = __fmul2_rn(u01, s1);
                        uint2 q0, q1;
                        q0.x = pack2(__ffma2_rn(u00, c0, __fmul2_rn(u10, s0)));
                        q0.y = pack2(__ffma2_rn(u01, c1, __fmul2_rn(u11, s1)));
                        q1.x = pack2(__ffma2_rn(u10, c0, make_float2(-t00.x, -t00.y)));
                        q1.y = pack2(__ffma2_rn(u11, c1, make_float2(-t01.x, -t01.y)));
                        *reinterpret_cast<uint2*>(base + o) = q0;
                        *reinterpret_cast<uint2*>(base + Cfg::SLAB + o) = q1;
                    }
                }
            }
            // exact mode: X' = diag(dw) X, in the chunk's theta stage once every rotation
            // thread is done with theta (R = 1), else in the X' buffer once dH of the previous
            // chunk has read it (in the scaled mode dH reads X itself)
            if (exact) {
                if (lead) {
                    if (R > 1 && c > 0) fail = !pwait(&bars[B_XP_EMPTY + ((c - 1) & 1)], (c - 1) >> 1, &s_abort);
                    fail = fail || !pwait(&bars[B_X_FULL + st], c >> 1, &s_abort);
                }
                if (bar_sync_or(1, kRThreads, fail || s_abort)) break;   // (R = 1: theta is consumed)
                const uint8_t* sX = sm + Cfg::X0 + st * Cfg::X_STAGE;
                uint8_t* sXP = sm + Cfg::xp(st);
                const float cend2 = sc[SC_MISC + MISC_CEND2];
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int item = (tid - kRWarp0 * 32) + it * kRThreads;
                    const int tr = (item >> 3) / R;   // dw = e^{cum_end - cum} w (0 past the end)
                    const float dw = ex2_approx(fminf(cend2 - sc[SC_A1 + tr], 0.f)) * sc[SC_A2 + tr];
                    const float2 dw2 = make_float2(dw, dw);
                    const uint32_t o = static_cast<uint32_t>(item) << 4;   // row * 128 + chunk * 16
                    const uint4 v = *reinterpret_cast<const uint4*>(sX + o);
                    uint4 r4;
                    r4.x = pack2_alu(__fmul2_rn(unpack2(v.x), dw2));
                    r4.y = pack2_alu(__fmul2_rn(unpack2(v.y), dw2));
                    r4.z = pack2_alu(__fmul2_rn(unpack2(v.z), dw2));
                    r4.w = pack2_alu(__fmul2_rn(unpack2(v.w), dw2));
                    *reinterpret_cast<uint4*>(sXP + o) = r4;
                }
            }
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_TH_EMPTY + st]);
                mbar_arrive(&bars[B_OPS + st]);
                mbar_arrive(&bars[B_SC_FREE + sb3]);
            }
        }
        // final angle (the sequence's cumulative angle, unreduced)
        if (last_seg && !s_abort && p.phi1) {
#pragma unroll
            for (int i = 0; i < 4; ++i) p.phi1[u * kHalf + 4 * j + i] = s_phi[4 * j + i];
        }
    } else if (warp < kTWarps) {
        // ================= TMEM warps =================
        const int trow = nrow;            // S / y row: (token, rank) = (trow / R, trow % R)
        const int tk = trow / R, rr = trow % R;
        const bool tlead = (warp == kTWarp0 && lane == 0);   // waits for the group
        auto tsync = [&](bool fail) { return !bar_sync_or(2, kTWarps * 32, fail || s_abort); };
        auto epilogue = [&](int c) {     // y of chunk c from its accumulator
            if (!tsync(tlead && !pwait(&bars[B_YD_FULL], c, &s_abort))) return false;
            fence_after_sync();
            const bool valid = c * Q + tk < L;
            __nv_bfloat16* dst = yu + static_cast<int64_t>(c * Q + tk) * tokY + rr * kP;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                float yv[32];
                tmem_ld_32x32b_x32(tmem + lanebase + T_Y + 64u * (c & 1) + 32u * hf, yv);
                tmem_wait_ld();
                if (hf == 1) {
                    fence_before_sync();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bars[B_Y_FREE + (c & 1)]);
                }
                if (valid) {
#pragma unroll
                    for (int q8 = 0; q8 < 4; ++q8) {
                        uint4 w;
                        w.x = pack_bf16(yv[8 * q8 + 0], yv[8 * q8 + 1]);
                        w.y = pack_bf16(yv[8 * q8 + 2], yv[8 * q8 + 3]);
                        w.z = pack_bf16(yv[8 * q8 + 4], yv[8 * q8 + 5]);
                        w.w = pack_bf16(yv[8 * q8 + 6], yv[8 * q8 + 7]);
                        *reinterpret_cast<uint4*>(dst + 32 * hf + 8 * q8) = w;
                    }
                }
            }
            return true;
        };
        bool ok = nchunks > 0 && tsync(tlead && !pwait(&bars[B_SC_READY], 0, &s_abort));
        if (ok) state_pass(1.f, s_sc, false);   // sigma H0 and the H0 operand of chunk 0
        // the loop and the final epilogue follow the group's votes only (every warp of the
        // group takes the same named barriers)
        for (int c = 0; c < nchunks && ok; ++c) {
            const int sb3 = c % kScBufs, sn3 = (c + 1) % kScBufs;
            const float* sc = s_sc + sb3 * SC_FLOATS;
            // S'(c), Yo(c) and dH(c) are done (one commit after all three); the scalars of
            // chunks c and c + 1
            const bool more = c + 1 < nchunks;
            bool fail = false;
            if (tlead) fail = !pwait(&bars[B_SD_FULL], c, &s_abort) ||
                              !pwait(&bars[B_SC_READY + sb3], c / kScBufs, &s_abort) ||
                              (more && !pwait(&bars[B_SC_READY + sn3], (c + 1) / kScBufs, &s_abort));
            if (!(ok = tsync(fail))) break;
            fence_after_sync();
            // ---- the state after chunk c: the next chunk's sigma H and H0, or the final state ----
            state_pass(sc[SC_MISC + MISC_XS], s_sc + sn3 * SC_FLOATS, !more);
            // ---- y of the previous chunk (its accumulator is read before P(c) is released) ----
            if (c > 0 && !(ok = epilogue(c - 1))) break;
            // ---- P into TMEM (bf16), 32-column blocks; blocks above the diagonal are zero ----
            const bool exact = sc[SC_MISC + MISC_MODE] != 0.f;
            const float gw = sc[SC_GW + tk];
            const float c2t = sc[SC_A1 + tk];   // log2-scaled cum (exact mode)
#pragma unroll 1
            for (int kb = 0; kb < 4; ++kb) {
                uint32_t pk[16];
                if (kb > tq) {
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = 0u;
                } else {
                    float v[32];
                    tmem_ld_32x32b_x32(tmem + lanebase + T_S + 128u * (c & 1) + 32u * kb, v);
                    tmem_wait_ld();
                    if (!exact) {
                        if (kb == tq) {   // the diagonal block: s < t kept, s = t weighted
#pragma unroll
                            for (int i = 0; i < 32; ++i) {
                                const int stok = (32 * kb + i) / R;
                                v[i] = (stok < tk) ? v[i] : ((stok == tk) ? v[i] * gw : 0.f);
                            }
                        }
                    } else {         // unit scales: the decay and weight element by element
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int stok = (32 * kb + i) / R;
                            const float m = (stok < tk) ? ex2_approx(fminf(c2t - sc[SC_A1 + stok], 0.f)) * sc[SC_A2 + stok]
                                                        : ((stok == tk) ? gw : 0.f);
                            v[i] *= m;
                        }
                    }
#pragma unroll
                    for (int i = 0; i < 16; ++i) pk[i] = pack_bf16(v[2 * i], v[2 * i + 1]);
                }
                tmem_st_32x32b_x16(tmem + lanebase + T_P + 16u * kb, pk);
            }
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_S_FREE + (c & 1)]);   // S'(c) has been read
            // ---- exact mode: the rows of Yo(c) times e^{cum_t} ----
            if (exact) {
                const float e = ex2_approx(c2t);
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    float yv[32];
                    const uint32_t ta = tmem + lanebase + T_Y + 64u * (c & 1) + 32u * hf;
                    tmem_ld_32x32b_x32(ta, yv);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 2; ++q) {
                        uint32_t w[16];
#pragma unroll
                        for (int i = 0; i < 16; ++i) w[i] = __float_as_uint(yv[16 * q + i] * e);
                        tmem_st_32x32b_x16(ta + 16u * q, w);
                    }
                }
            }
            tmem_wait_st();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bars[B_P_FULL]);
                mbar_arrive(&bars[B_SC_FREE + sb3]);
            }
        }
        if (ok && nchunks > 0) ok = epilogue(nchunks - 1);
    } else if (warp == kMmaWarp) {
        // ================= S', Yo and dH issue (one lane) =================
        // Per chunk c: S'(c) once the rotation warps are done with chunk c and S' buffer c & 1
        // is free; Yo(c) and dH(c) once the state pass of chunk c-1 has written H0 and sigma H;
        // then one commit for all three. Yd is issued by the next warp, so that a chunk's mask
        // never holds up the next chunk's products.
        if (lane == 0) {
            constexpr uint32_t hi = desc_hi_sw128(1024);
            constexpr uint32_t id_s = idesc_bf16(128, 128, false, false);   // S' = C' . B'^T
            constexpr uint32_t id_dh = idesc_bf16(128, 64, true, true);     // dH = B'^T . X
            constexpr uint32_t id_y = idesc_bf16(128, 64, false, true);     // Y = C' . H0
            const uint32_t loH = desc_lo(smem_u32(sm + Cfg::H0), 16384);
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                if (!pwait(&bars[B_OPS + st], c >> 1, &s_abort)) break;
                if (c >= 2 && !pwait(&bars[B_S_FREE + st], (c >> 1) - 1, &s_abort)) break;
                fence_after_sync();
                const uint32_t aB = smem_u32(sm + st * Cfg::BC_STAGE), aC = aB + Cfg::C_OFF;
                const uint32_t loB = desc_lo(aB, 16), loC = desc_lo(aC, 16);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tmem + T_S + 128u * st, desc_pack(loC + (kmajor_off(k, Cfg::SLAB) >> 4), hi),
                             desc_pack(loB + (kmajor_off(k, Cfg::SLAB) >> 4), hi), id_s, k > 0);
                issued = 1;
                if (!pwait(&bars[B_H0_FULL], c, &s_abort) || !pwait(&bars[B_DH_FREE], c, &s_abort) ||
                    !pwait(&bars[B_X_FULL + st], c >> 1, &s_abort) ||
                    (c >= 2 && !pwait(&bars[B_Y_FREE + st], (c >> 1) - 1, &s_abort)))
                    break;
                fence_after_sync();
                const bool exact = s_sc[(c % kScBufs) * SC_FLOATS + SC_MISC + MISC_MODE] != 0.f;
                const uint32_t loBt = desc_lo(aB, Cfg::SLAB);
                const uint32_t loDX = desc_lo(smem_u32(sm + (exact ? Cfg::xp(st) : Cfg::X0 + st * Cfg::X_STAGE)), 16384);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tmem + T_Y + 64u * st, desc_pack(loC + (kmajor_off(k, Cfg::SLAB) >> 4), hi),
                             desc_pack(loH + (mnmajor_off(k) >> 4), hi), id_y, k > 0);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16(tmem + T_H, desc_pack(loBt + (mnmajor_off(k) >> 4), hi),
                             desc_pack(loDX + (mnmajor_off(k) >> 4), hi), id_dh, 1u);
                mma_commit(smem_u32(&bars[B_SD_FULL]));
                mma_commit(smem_u32(&bars[B_XP_EMPTY + st]));
                mma_commit(smem_u32(&bars[B_BC_EMPTY + st]));
            }
            if (s_abort && issued) {   // let this CTA's MMAs finish before TMEM is released
                mma_commit(smem_u32(&bars[B_DRAIN]));
                (void)mbar_wait(&bars[B_DRAIN], 0, 200000000LL);
            }
        }
        __syncwarp();
    } else if (warp == kYdWarp) {
        // ================= Yd issue (one lane) =================
        // Yd(c) = P(c) X(c) onto Yo(c), once P(c) is in TMEM (which the TMEM warps write after
        // S'(c), Yo(c) and dH(c) are done).
        if (lane == 0) {
            constexpr uint32_t hi = desc_hi_sw128(1024);
            constexpr uint32_t id_y = idesc_bf16(128, 64, false, true);     // Y += P . X
            int issued = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                if (!pwait(&bars[B_P_FULL], c, &s_abort)) break;
                fence_after_sync();
                const uint32_t loX = desc_lo(smem_u32(sm + Cfg::X0 + st * Cfg::X_STAGE), 16384);
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    mma_bf16_ts(tmem + T_Y + 64u * st, tmem + T_P + 8u * k,
                                desc_pack(loX + (mnmajor_off(k) >> 4), hi), id_y, 1u);
                mma_commit(smem_u32(&bars[B_YD_FULL]));
                mma_commit(smem_u32(&bars[B_X_EMPTY + st]));
                issued = 1;
            }
            if (s_abort && issued) {
                mma_commit(smem_u32(&bars[B_DRAIN2]));
                (void)mbar_wait(&bars[B_DRAIN2], 0, 200000000LL);
            }
        }
        __syncwarp();
    } else if (warp == kLoadWarp) {
        // ================= TMA loads (one lane) =================
        if (lane == 0) {
            int n_th0 = 0, n_th1 = 0, n_bc0 = 0, n_bc1 = 0, n_x0 = 0, n_x1 = 0;   // loads issued
            for (int c = 0; c < nchunks; ++c) {
                const int st = c & 1;
                // theta into its stage once chunk c-2 is done with it (the walk, and dH reading
                // X' where the exact mode put it there)
                if (c >= 2 && (!pwait(&bars[B_TH_EMPTY + st], (c >> 1) - 1, &s_abort) ||
                               !pwait(&bars[B_XP_EMPTY + st], (c >> 1) - 1, &s_abort)))
                    break;
                if (!(blockIdx.x == 0 && c > 0 && c == p.test_skip_theta)) {   // (test hook)
                    mbar_arrive_expect_tx(&bars[B_TH_FULL + st], Cfg::TH_TX);
                    tma_load_4d(sm + Cfg::TH0 + st * Cfg::TH_STAGE, &maps.theta,
                                &bars[B_TH_FULL + st], 0, ih, c * Q, ib);
                    if (st) ++n_th1; else ++n_th0;
                }
                if (c >= 2 && !pwait(&bars[B_BC_EMPTY + st], (c >> 1) - 1, &s_abort)) break;
                uint64_t* bar = &bars[B_BC_FULL + st];
                mbar_arrive_expect_tx(bar, Cfg::BC_TX + (rsu ? kRows * 8u : 0u));
                uint8_t* base = sm + st * Cfg::BC_STAGE;
                tma_load_5d(base, &maps.B, bar, 0, 0, ig, c * Q, ib);
                tma_load_5d(base + Cfg::SLAB, &maps.B, bar, kHalf, 0, ig, c * Q, ib);
                tma_load_5d(base + Cfg::C_OFF, &maps.C, bar, 0, 0, ig, c * Q, ib);
                tma_load_5d(base + Cfg::C_OFF + Cfg::SLAB, &maps.C, bar, kHalf, 0, ig, c * Q, ib);
                if (rsu && c == 0) grid_dep_wait();   // the scales' kernel may still run
                if (rsu) bulk_load(sm + Cfg::RS + st * (kRows * 8), rsu + static_cast<int64_t>(c) * Q * R,
                                   kRows * 8u, bar);
                if (st) ++n_bc1; else ++n_bc0;
                if (c >= 2 && !pwait(&bars[B_X_EMPTY + st], (c >> 1) - 1, &s_abort)) break;
                mbar_arrive_expect_tx(&bars[B_X_FULL + st], Cfg::X_TX);
                tma_load_5d(sm + Cfg::X0 + st * Cfg::X_STAGE, &maps.x, &bars[B_X_FULL + st], 0, 0,
                            ih, c * Q, ib);
                if (st) ++n_x1; else ++n_x0;
            }
            {   // every copy issued has landed before the CTA exits (at once unless a wait
                // elsewhere gave up while copies were in flight)
                constexpr long long kDrain = 200000000LL;
                if (n_th0 > 0) (void)mbar_wait(&bars[B_TH_FULL], (n_th0 - 1) & 1, kDrain);
                if (n_th1 > 0) (void)mbar_wait(&bars[B_TH_FULL1], (n_th1 - 1) & 1, kDrain);
                if (n_bc0 > 0) (void)mbar_wait(&bars[B_BC_FULL], (n_bc0 - 1) & 1, kDrain);
                if (n_bc1 > 0) (void)mbar_wait(&bars[B_BC_FULL1], (n_bc1 - 1) & 1, kDrain);
                if (n_x0 > 0) (void)mbar_wait(&bars[B_X_FULL], (n_x0 - 1) & 1, kDrain);
                if (n_x1 > 0) (void)mbar_wait(&bars[B_X_FULL1], (n_x1 - 1) & 1, kDrain);
            }
        }
        __syncwarp();
    } else {
        // ================= chunk scalars (whole warp) =================
        // raw dt, A, lam of chunk c in registers: TPL tokens per lane, and the chunk's
        // look-ahead token (the next chunk's first)
        float rdt[TPL], rA[TPL], rlm[TPL], rdt_n = 0.f, rlm_n = 0.f;
        auto fetch = [&](int c) {
            const int64_t base = bb * p.L * p.H + hh;
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int t = c * Q + lane * TPL + i;
                const bool v = t < L;
                const int64_t idx = base + static_cast<int64_t>(t) * p.H;
                rdt[i] = v ? __ldg(p.dt + idx) : 0.f;
                rA[i] = v ? __ldg(p.A + idx) : 0.f;
                rlm[i] = v ? __ldg(p.lam + idx) : 0.f;
            }
            const int tn = (c + 1) * Q;
            const int64_t idn = base + static_cast<int64_t>(tn) * p.H;
            rdt_n = (tn < L) ? __ldg(p.dt + idn) : 0.f;
            rlm_n = (tn < L) ? __ldg(p.lam + idn) : 0.f;
        };
        auto scalars = [&](int c) {
            float* blk = s_sc + (c % kScBufs) * SC_FLOATS;
            const int c0 = c * Q;
            const int T = (L - c0) < Q ? (L - c0) : Q;
            const bool zoh = kRaw && (p.flags & 4u);
            float d[TPL], a[TPL], lm[TPL], ga[TPL], w[TPL];
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const bool v = lane * TPL + i < T;
                d[i] = v ? step_dt<kRaw>(rdt[i], dtb, p.flags) : 0.f;
                lm[i] = v ? step_lam<kRaw>(rlm[i], p.flags) : 0.f;
                a[i] = d[i] * rA[i];
                ga[i] = lm[i] * d[i];
            }
            // the next token's (1 - lam) dt: same lane, the next lane's first token, or (lane
            // 31) the look-ahead token; zero past the sequence end
            float dn = __shfl_down_sync(0xffffffffu, d[0], 1);
            float ln = __shfl_down_sync(0xffffffffu, lm[0], 1);
            if (lane == 31) {
                const bool v = c0 + Q < L;
                dn = v ? step_dt<kRaw>(rdt_n, dtb, p.flags) : 0.f;
                ln = v ? step_lam<kRaw>(rlm_n, p.flags) : 0.f;
            }
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const float dnx = (i + 1 < TPL) ? d[(i + 1) % TPL] : dn;
                const float lnx = (i + 1 < TPL) ? lm[(i + 1) % TPL] : ln;
                w[i] = ga[i] + (1.f - lnx) * dnx;
                if (zoh) {
                    const bool v = lane * TPL + i < T;
                    ga[i] = v ? zoh_gamma(d[i], rA[i]) : 0.f;
                    w[i] = ga[i];
                }
            }
            float cl[TPL], s = 0.f;
#pragma unroll
            for (int i = 0; i < TPL; ++i) { s += a[i]; cl[i] = s; }
            const float incl = warp_inclusive_scan(s);
            const float excl = incl - s;
            // cum at the chunk's last real token T - 1
            float mine = 0.f;
#pragma unroll
            for (int i = 0; i < TPL; ++i) if (((T - 1) % TPL) == i) mine = excl + cl[i];
            const float cum_end = __shfl_sync(0xffffffffu, mine, (T - 1) / TPL);
            float cm[TPL];
#pragma unroll
            for (int i = 0; i < TPL; ++i) cm[i] = (lane * TPL + i < T) ? excl + cl[i] : cum_end;
            // the chunk's reference: the midpoint of cum over its real tokens; the scaled mode
            // when the chunk decays by at most kMaxChunkDecay
            const float first = __shfl_sync(0xffffffffu, cm[0], 0);
            const float ref = 0.5f * (first + cum_end);
            const bool exact = first - cum_end > kMaxChunkDecay;
            constexpr float kLog2e = 1.4426950408889634f;
#pragma unroll
            for (int i = 0; i < TPL; ++i) {
                const int t = lane * TPL + i;
                const bool v = t < T;
                blk[SC_DT + t] = d[i];
                if (!exact) {
                    blk[SC_A1 + t] = __expf(ref - cm[i]) * w[i];
                    blk[SC_A2 + t] = __expf(cm[i] - ref);
                    blk[SC_GW + t] = w[i] > 0.f ? __fdividef(ga[i], w[i]) : 0.f;
                } else {
                    blk[SC_A1 + t] = cm[i] * kLog2e;
                    blk[SC_A2 + t] = v ? w[i] : 0.f;
                    blk[SC_GW + t] = ga[i];
                }
            }
            if (lane == 0) {
                blk[SC_MISC + MISC_EEND] = __expf(cum_end);
                blk[SC_MISC + MISC_MODE] = exact ? 1.f : 0.f;
                blk[SC_MISC + MISC_XS] = exact ? 1.f : __expf(cum_end - ref);
                blk[SC_MISC + MISC_EH0] = exact ? 1.f : __expf(ref);
                blk[SC_MISC + MISC_CEND2] = cum_end * kLog2e;
            }
        };
        if (nchunks > 0) fetch(0);
        for (int c = 0; c < nchunks && !s_abort; ++c) {
            const int sb3 = c % kScBufs;
            if (c >= kScBufs && !pwait(&bars[B_SC_FREE + sb3], c / kScBufs - 1, &s_abort)) break;
            scalars(c);
            __syncwarp();
            if (lane == 0) mbar_arrive(&bars[B_SC_READY + sb3]);
            if (c + 1 < nchunks) fetch(c + 1);
        }
    }

    // ---------------- final state ----------------
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    if (!s_abort && L > 0) {
        if (p.prevB1) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevB1) + u * R * kN;
            const __nv_bfloat16* src = Bu + static_cast<int64_t>(L - 1) * tokB;
            for (int e = tid; e < R * kN; e += kThreads) dst[e] = src[e];
        }
        if (p.prevx1) {
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.prevx1) + u * R * kP;
            const __nv_bfloat16* src = xu + static_cast<int64_t>(L - 1) * tokY;
            for (int e = tid; e < R * kP; e += kThreads) dst[e] = src[e];
        }
    }
    if (s_abort && tid == 0 && p.status) atomicExch(p.status, 1);
    if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
        return static_cast<PFN_cuTensorMapEncodeTiled_v12000>(nullptr);
    }();
    return fn;
}

bool encode_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box) {
    auto enc = encode_fn();
    if (!enc) return false;
    const cuuint32_t es[5] = {1, 1, 1, 1, 1};
    return enc(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t pipe_rs_bytes(const ScanParams& p) {
    const int64_t Q = kRows / (p.R > 0 ? p.R : 1);
    const int64_t Lpad = (p.L + Q - 1) / Q * Q;
    const size_t n = p.bc_norm ? static_cast<size_t>(p.b * Lpad * p.G * p.R) * sizeof(float2) : 0;
    return (n + 255) / 256 * 256;
}

template <int R, bool kRaw>
cudaError_t launch_pipe_t(const ScanParams& p, float2* rs, cudaStream_t s) {
    constexpr int Q = PCfg<R>::Q;
    PMaps maps;
    const cuuint64_t H = p.H, Lq = p.L, b = p.b, Gq = p.G;
    {   // x [b][L][H][R][P], box (P, R, 1, Q, 1): 128 rows of 128 bytes
        const cuuint64_t dims[5] = {kP, static_cast<cuuint64_t>(R), H, Lq, b};
        const cuuint64_t str[4] = {kP * 2, R * kP * 2, H * R * kP * 2, Lq * H * R * kP * 2};
        const cuuint32_t box[5] = {kP, static_cast<cuuint32_t>(R), 1, Q, 1};
        if (!encode_map(&maps.x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.x, dims, str, box))
            return cudaErrorInvalidValue;
    }
    {   // theta [b][L][H][N/2], box (64, 1, Q, 1)
        const cuuint64_t dims[4] = {kHalf, H, Lq, b};
        const cuuint64_t str[3] = {kHalf * 2, H * kHalf * 2, Lq * H * kHalf * 2};
        const cuuint32_t box[4] = {kHalf, 1, Q, 1};
        if (!encode_map(&maps.theta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, p.theta, dims, str, box))
            return cudaErrorInvalidValue;
    }
    {   // B, C [b][L][G][R][N], box (64 columns, R, 1, Q, 1): one 64-column slab per load
        const cuuint64_t dims[5] = {kN, static_cast<cuuint64_t>(R), Gq, Lq, b};
        const cuuint64_t str[4] = {kN * 2, R * kN * 2, Gq * R * kN * 2, Lq * Gq * R * kN * 2};
        const cuuint32_t box[5] = {kHalf, static_cast<cuuint32_t>(R), 1, Q, 1};
        if (!encode_map(&maps.B, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.B, dims, str, box) ||
            !encode_map(&maps.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, p.C, dims, str, box))
            return cudaErrorInvalidValue;
    }
    if (rs) {
        cudaError_t e = launch_rms_scales(p, Q, rs, s);
        if (e != cudaSuccess) return e;
    }
    auto k = scan_pipe_kernel<R, kRaw>;
    const uint32_t smem = PCfg<R>::SMEM;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (rs)   // may start while the scales' kernel finishes (the TMA lane waits for it)
        return launch_after_rms(k, static_cast<unsigned>(p.b * p.H), kThreads, smem, s, p, maps,
                                static_cast<const float2*>(rs));
    k<<<static_cast<unsigned>(p.b * p.H), kThreads, smem, s>>>(p, maps, rs);
    return cudaGetLastError();
}

}  // namespace

bool pipe_scan_supported(const ScanParams& p, bool bf16) {
    // 32-bit element offsets inside one sequence: L * G * R * N and L * H * R * P < 2^31
    const int64_t lim = 0x7fffffffLL;
    return bf16 && p.N == kN && p.P == kP && p.Q * p.R == kRows &&
           (p.R == 1 || p.R == 2 || p.R == 4) && p.L * p.G * p.R * kN < lim &&
           p.L * p.H * p.R * kP < lim && p.b * p.H <= lim;
}

size_t pipe_scan_workspace_bytes(const ScanParams& p) { return pipe_rs_bytes(p); }

cudaError_t launch_scan_pipe(const ScanParams& p_in, void* ws_body, size_t body_bytes, cudaStream_t s) {
    if (p_in.b * p_in.H == 0 || p_in.L == 0) return cudaSuccess;
    ScanParams p = p_in;
    if (const char* e = std::getenv("M3_TEST_SKIP_THETA_LOAD")) p.test_skip_theta = std::atoi(e);
    float2* rs = p.bc_norm ? static_cast<float2*>(ws_body) : nullptr;
    if (body_bytes < pipe_rs_bytes(p)) return cudaErrorInvalidValue;
    const bool raw = p.flags != 0;
    switch (p.R) {
        case 1: return raw ? launch_pipe_t<1, true>(p, rs, s) : launch_pipe_t<1, false>(p, rs, s);
        case 2: return raw ? launch_pipe_t<2, true>(p, rs, s) : launch_pipe_t<2, false>(p, rs, s);
        case 4: return raw ? launch_pipe_t<4, true>(p, rs, s) : launch_pipe_t<4, false>(p, rs, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace m3
