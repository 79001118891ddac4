// Host side of the C ABI declared in include/m3.h: argument validation, workspace layout and
// dispatch to the kernels. Nothing here allocates device memory or synchronises a stream
// (m3_scan_check excepted, which is documented to block).
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "m3_internal.h"

namespace m3 {
namespace {

thread_local char g_err[512] = "";

m3_status fail(m3_status s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

m3_status cuda_fail(cudaError_t e, const char* where) {
    return fail(M3_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kWsHeader = 256;  // status word + padding

m3_status check_dims(const m3_dims* d, bool scan) {
    if (!d) return fail(M3_ERR_INVALID_ARG, "dims is NULL");
    if (d->in_dtype != M3_F32 && d->in_dtype != M3_BF16)
        return fail(M3_ERR_INVALID_ARG, "in_dtype %d is not M3_F32 or M3_BF16", d->in_dtype);
    if (d->batch < 0 || d->seqlen < 0)
        return fail(M3_ERR_INVALID_ARG, "batch and seqlen must be >= 0");
    if (d->nheads < 1 || d->ngroups < 1 || d->nheads % d->ngroups != 0)
        return fail(M3_ERR_INVALID_ARG, "nheads (%lld) must be a positive multiple of ngroups (%lld)",
                    (long long)d->nheads, (long long)d->ngroups);
    if (d->headdim < 1 || d->dstate < 2 || d->dstate % 2 != 0 || d->rank < 1)
        return fail(M3_ERR_INVALID_ARG, "headdim >= 1, even dstate >= 2 and rank >= 1 required");
    if (!(d->norm_eps >= 0.f) || !std::isfinite(d->norm_eps))
        return fail(M3_ERR_INVALID_ARG, "norm_eps must be finite and >= 0");
    if (d->flags & ~(M3_DT_SOFTPLUS | M3_LAM_SIGMOID | M3_DISC_ZOH | M3_BWD_FP32))
        return fail(M3_ERR_INVALID_ARG, "unknown bits in flags (0x%x)", (unsigned)d->flags);
    if (d->headdim != 16 && d->headdim != 32 && d->headdim != 64 && d->headdim != 128)
        return fail(M3_ERR_UNSUPPORTED, "headdim %lld not in {16, 32, 64, 128}",
                    (long long)d->headdim);
    if (d->dstate % 16 != 0 || d->dstate > 256)
        return fail(M3_ERR_UNSUPPORTED, "dstate %lld must be a multiple of 16 and <= 256",
                    (long long)d->dstate);
    if (d->rank != 1 && d->rank != 2 && d->rank != 4 && d->rank != 8)
        return fail(M3_ERR_UNSUPPORTED, "rank %lld not in {1, 2, 4, 8}", (long long)d->rank);
    if (scan) {
        if (d->chunk < 1) return fail(M3_ERR_INVALID_ARG, "chunk must be >= 1");
        if (d->chunk * d->rank > 128)
            return fail(M3_ERR_UNSUPPORTED, "chunk * rank = %lld exceeds 128",
                        (long long)(d->chunk * d->rank));
    }
    if (d->batch * d->nheads > (int64_t)0x7fffffff)
        return fail(M3_ERR_UNSUPPORTED, "batch * nheads exceeds the grid limit");
    return M3_OK;
}

m3_status check_inputs(const m3_inputs* in, bool need) {
    if (!in) return fail(M3_ERR_INVALID_ARG, "inputs is NULL");
    if (!need) return M3_OK;
    const void* req[] = {in->x, in->B, in->C, in->theta, in->dt, in->A, in->lam};
    const char* names[] = {"x", "B", "C", "theta", "dt", "A", "lam"};
    for (int i = 0; i < 7; ++i) {
        if (!req[i]) return fail(M3_ERR_INVALID_ARG, "input %s is NULL", names[i]);
        if (!aligned16(req[i]))
            return fail(M3_ERR_INVALID_ARG, "input %s is not 16-byte aligned", names[i]);
    }
    if (in->B_bias && !aligned16(in->B_bias)) return fail(M3_ERR_INVALID_ARG, "B_bias misaligned");
    if (in->C_bias && !aligned16(in->C_bias)) return fail(M3_ERR_INVALID_ARG, "C_bias misaligned");
    if (in->dt_bias && (reinterpret_cast<uintptr_t>(in->dt_bias) & 3u) != 0)
        return fail(M3_ERR_INVALID_ARG, "dt_bias misaligned");
    return M3_OK;
}

m3_status check_state(const m3_state* s, const char* what) {
    if (!s) return M3_OK;
    const void* f[] = {s->h, s->phi, s->prev_B, s->prev_x};
    const char* names[] = {"h", "phi", "prev_B", "prev_x"};
    for (int i = 0; i < 4; ++i) {
        if (!f[i]) return fail(M3_ERR_INVALID_ARG, "%s state field %s is NULL", what, names[i]);
        if (!aligned16(f[i]))
            return fail(M3_ERR_INVALID_ARG, "%s state field %s is not 16-byte aligned", what, names[i]);
    }
    return M3_OK;
}

ScanParams make_params(const m3_dims* d, const m3_inputs* in, const m3_state* init,
                       const m3_state* fin, void* y) {
    ScanParams p{};
    p.b = d->batch; p.L = d->seqlen; p.H = d->nheads; p.G = d->ngroups; p.P = d->headdim;
    p.N = d->dstate; p.R = d->rank; p.Q = d->chunk;
    p.bc_norm = d->bc_norm ? 1 : 0; p.eps = d->norm_eps;
    p.x = in->x; p.B = in->B; p.C = in->C; p.theta = in->theta;
    p.dt = in->dt; p.A = in->A; p.lam = in->lam; p.Bbias = in->B_bias; p.Cbias = in->C_bias;
    p.dt_bias = in->dt_bias; p.flags = d->flags & ~M3_BWD_FP32;   // a choice of path, not of scalars
    if (init) { p.h0 = init->h; p.phi0 = init->phi; p.prevB0 = init->prev_B; p.prevx0 = init->prev_x; }
    if (fin) { p.h1 = fin->h; p.phi1 = fin->phi; p.prevB1 = fin->prev_B; p.prevx1 = fin->prev_x; }
    p.y = y;
    return p;
}

size_t elem_size(const m3_dims* d) { return d->in_dtype == M3_BF16 ? 2 : 4; }

// Sequence of length 0: the final state is the initial one (or zeros).
m3_status empty_sequence(const m3_dims* d, const m3_state* init, const m3_state* fin,
                         cudaStream_t s) {
    if (!fin) return M3_OK;
    const size_t u = static_cast<size_t>(d->batch * d->nheads);
    const size_t bytes[4] = {u * d->dstate * d->headdim * 4, u * (d->dstate / 2) * 4,
                             u * d->rank * d->dstate * elem_size(d),
                             u * d->rank * d->headdim * elem_size(d)};
    void* dst[4] = {fin->h, fin->phi, fin->prev_B, fin->prev_x};
    const void* src[4] = {init ? init->h : nullptr, init ? init->phi : nullptr,
                          init ? init->prev_B : nullptr, init ? init->prev_x : nullptr};
    for (int i = 0; i < 4; ++i) {
        if (bytes[i] == 0) continue;
        cudaError_t e = src[i] ? (src[i] == dst[i] ? cudaSuccess
                                                   : cudaMemcpyAsync(dst[i], src[i], bytes[i],
                                                                     cudaMemcpyDeviceToDevice, s))
                               : cudaMemsetAsync(dst[i], 0, bytes[i], s);
        if (e != cudaSuccess) return cuda_fail(e, "empty-sequence state copy");
    }
    return M3_OK;
}

}  // namespace

m3_status set_error(m3_status s, const char* msg) { return fail(s, "%s", msg); }

int device_sm_count() {
    constexpr int kSlots = 64, kDefault = 148;
    static std::atomic<int> cached[kSlots];   // 0 until the device's count is known
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kSlots) return kDefault;
    int sms = cached[dev].load(std::memory_order_relaxed);
    if (sms > 0) return sms;
    // two threads may both look it up; they store the same value
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return kDefault;
    cached[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

}  // namespace m3

using namespace m3;

extern "C" {

size_t m3_scan_workspace_bytes(const m3_dims* dims) {
    if (check_dims(dims, true) != M3_OK) return 0;
    const m3_inputs none{};
    const ScanParams p = make_params(dims, &none, nullptr, nullptr, nullptr);
    size_t body = 0;
    if (pipe_scan_supported(p, dims->in_dtype == M3_BF16)) body = pipe_scan_workspace_bytes(p);
    else if (tc_scan_supported(p, dims->in_dtype == M3_BF16)) body = tc_scan_workspace_bytes(p);
    return kWsHeader + (body + 255) / 256 * 256;
}

}  // extern "C"

namespace m3 {

// The smallest workspace the scan runs in: without the sequence-parallel form's segment
// states (0 for invalid dims).
size_t scan_workspace_min_bytes(const m3_dims* dims) {
    if (check_dims(dims, true) != M3_OK) return 0;
    const m3_inputs none{};
    const ScanParams p = make_params(dims, &none, nullptr, nullptr, nullptr);
    size_t body = 0;
    if (pipe_scan_supported(p, dims->in_dtype == M3_BF16)) body = pipe_scan_workspace_bytes(p);
    else if (tc_scan_supported(p, dims->in_dtype == M3_BF16)) body = tc_scan_workspace_min_bytes(p);
    return kWsHeader + (body + 255) / 256 * 256;
}

// m3_scan_fwd with the workspace size it must at least have (`need`).
m3_status scan_fwd_with(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                        const m3_state* final_state, void* y, void* workspace, size_t ws_bytes,
                        size_t need, void* stream) {
    g_err[0] = 0;
    m3_status st = check_dims(dims, true);
    if (st != M3_OK) return st;
    const bool any = dims->batch * dims->seqlen * dims->nheads > 0;
    if ((st = check_inputs(in, any)) != M3_OK) return st;
    if ((st = check_state(init, "initial")) != M3_OK) return st;
    if ((st = check_state(final_state, "final")) != M3_OK) return st;
    if (any && !y) return fail(M3_ERR_INVALID_ARG, "y is NULL");
    if (y && !aligned16(y)) return fail(M3_ERR_INVALID_ARG, "y is not 16-byte aligned");
    if (!workspace) return fail(M3_ERR_INVALID_ARG, "workspace is NULL");
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return fail(M3_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
    if (ws_bytes < need)
        return fail(M3_ERR_INVALID_ARG, "workspace has %zu bytes, %zu needed", ws_bytes, need);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    ScanParams p = make_params(dims, in, init, final_state, y);
    p.ws = workspace;
    p.ws_bytes = ws_bytes;
    p.status = static_cast<int32_t*>(workspace);
    cudaError_t e;
    if (dims->seqlen == 0 || dims->batch == 0) return empty_sequence(dims, init, final_state, s);

    const bool bf16 = dims->in_dtype == M3_BF16;
    if (pipe_scan_supported(p, bf16)) {
        e = launch_scan_pipe(p, static_cast<char*>(workspace) + kWsHeader, ws_bytes - kWsHeader, s);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core scan launch");
        return M3_OK;
    }
    if (tc_scan_supported(p, bf16)) {
        e = launch_scan_tc(p, static_cast<char*>(workspace) + kWsHeader, ws_bytes - kWsHeader, s);
        if (e != cudaSuccess) return cuda_fail(e, "tensor-core scan launch");
        return M3_OK;
    }
    const size_t smem = simt_scan_smem_bytes(p);
    if (smem > 227 * 1024)
        return fail(M3_ERR_UNSUPPORTED, "shape needs %zu bytes of shared memory", smem);
    e = launch_scan_simt(p, bf16, s);
    if (e != cudaSuccess) return cuda_fail(e, "scan launch");
    return M3_OK;
}

}  // namespace m3

extern "C" {

m3_status m3_scan_fwd(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                      const m3_state* final_state, void* y, void* workspace, size_t ws_bytes,
                      void* stream) {
    return scan_fwd_with(dims, in, init, final_state, y, workspace, ws_bytes,
                         m3_scan_workspace_bytes(dims), stream);
}

}  // extern "C"

namespace m3 {
namespace {

// m3_decode_step, with the MIMO projections when proj is not NULL (x then comes from proj).
m3_status decode_impl(const m3_dims* dims, const m3_inputs* in, const m3_proj* proj,
                      const m3_state* state_in, const m3_state* state_out, void* y, void* stream) {
    g_err[0] = 0;
    m3_status st = check_dims(dims, false);
    if (st != M3_OK) return st;
    if (dims->seqlen != 1) return fail(M3_ERR_INVALID_ARG, "decode needs seqlen == 1");
    if (!state_in || !state_out) return fail(M3_ERR_INVALID_ARG, "state_in and state_out are required");
    const bool any = dims->batch > 0;
    if (!in) return fail(M3_ERR_INVALID_ARG, "inputs is NULL");
    m3_inputs ins = *in;
    if (proj) {
        const void* req[] = {proj->x_in, proj->z_in, proj->W_X, proj->W_Z, proj->W_O};
        const char* names[] = {"x_in", "z_in", "W_X", "W_Z", "W_O"};
        for (int i = 0; i < 5 && any; ++i) {
            if (!req[i]) return fail(M3_ERR_INVALID_ARG, "projection %s is NULL", names[i]);
            if (!aligned16(req[i]))
                return fail(M3_ERR_INVALID_ARG, "projection %s is not 16-byte aligned", names[i]);
        }
        ins.x = proj->x_in;   // checked like x; the kernels read it as [b, H, P]
    }
    if ((st = check_inputs(&ins, any)) != M3_OK) return st;
    if ((st = check_state(state_in, "input")) != M3_OK) return st;
    if ((st = check_state(state_out, "output")) != M3_OK) return st;
    if (any && (!y || !aligned16(y))) return fail(M3_ERR_INVALID_ARG, "output is NULL or misaligned");
    if (!any) return M3_OK;
    ScanParams p = make_params(dims, &ins, state_in, state_out, y);
    if (proj) {
        p.proj = 1;
        p.xprj = proj->x_in;
        p.zprj = proj->z_in;
        p.WX = proj->W_X;
        p.WZ = proj->W_Z;
        p.WO = proj->W_O;
    }
    const size_t smem = decode_smem_bytes(p);
    if (smem > 227 * 1024) return fail(M3_ERR_UNSUPPORTED, "decode shape too large");
    cudaError_t e = launch_decode(p, dims->in_dtype == M3_BF16, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "decode launch");
    return M3_OK;
}

}  // namespace
}  // namespace m3

extern "C" {

m3_status m3_decode_step(const m3_dims* dims, const m3_inputs* in, const m3_state* state_in,
                         const m3_state* state_out, void* y, void* stream) {
    return decode_impl(dims, in, nullptr, state_in, state_out, y, stream);
}

m3_status m3_scan_state(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                        const m3_seg_state* out, void* workspace, size_t ws_bytes, void* stream) {
    g_err[0] = 0;
    m3_status st = check_dims(dims, true);
    if (st != M3_OK) return st;
    const bool any = dims->batch * dims->seqlen * dims->nheads > 0;
    if ((st = check_inputs(in, any)) != M3_OK) return st;
    if ((st = check_state(init, "initial")) != M3_OK) return st;
    if (!out || !out->h || !out->phi || !out->lam_sum)
        return fail(M3_ERR_INVALID_ARG, "out and its h, phi, lam_sum are required");
    if (!aligned16(out->h) || !aligned16(out->phi) || !aligned16(out->lam_sum))
        return fail(M3_ERR_INVALID_ARG, "out fields must be 16-byte aligned");
    const m3_inputs none{};
    const ScanParams q = make_params(dims, &none, nullptr, nullptr, nullptr);
    if (!tc_scan_supported(q, dims->in_dtype == M3_BF16))
        return fail(M3_ERR_UNSUPPORTED, "m3_scan_state runs the tensor-core shapes only");
    const size_t need = scan_workspace_min_bytes(dims);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < need)
        return fail(M3_ERR_INVALID_ARG, "workspace: NULL, misaligned or below %zu bytes", need);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t units = dims->batch * dims->nheads, N = dims->dstate, P = dims->headdim;
    if (units == 0) return M3_OK;
    if (dims->seqlen == 0) {   // no token: the initial state, nothing decayed
        cudaError_t e = init ? cudaMemcpyAsync(out->h, init->h, units * N * P * 4, cudaMemcpyDeviceToDevice, s)
                             : cudaMemsetAsync(out->h, 0, units * N * P * 4, s);
        if (e == cudaSuccess)
            e = init ? cudaMemcpyAsync(out->phi, init->phi, units * (N / 2) * 4, cudaMemcpyDeviceToDevice, s)
                     : cudaMemsetAsync(out->phi, 0, units * (N / 2) * 4, s);
        if (e == cudaSuccess) e = cudaMemsetAsync(out->lam_sum, 0, units * 4, s);
        return e == cudaSuccess ? M3_OK : cuda_fail(e, "empty segment copy");
    }
    ScanParams p = make_params(dims, in, init, nullptr, nullptr);
    p.ws = workspace;
    p.ws_bytes = ws_bytes;
    p.status = static_cast<int32_t*>(workspace);
    cudaError_t e = launch_scan_state_tc(p, static_cast<char*>(workspace) + kWsHeader,
                                         ws_bytes - kWsHeader, out->h, out->phi, out->lam_sum, s);
    if (e != cudaSuccess) return cuda_fail(e, "state-only scan launch");
    return M3_OK;
}

m3_status m3_state_combine(const m3_dims* dims, int nseg, const m3_seg_state* seg, float* h_out,
                           float* phi_out, void* stream) {
    g_err[0] = 0;
    m3_status st = check_dims(dims, false);
    if (st != M3_OK) return st;
    if (nseg < 1) return fail(M3_ERR_INVALID_ARG, "nseg must be >= 1");
    if (!seg || !seg->h || !seg->phi || !seg->lam_sum || !h_out || !phi_out)
        return fail(M3_ERR_INVALID_ARG, "seg fields, h_out and phi_out are required");
    const void* ptrs[] = {seg->h, seg->phi, seg->lam_sum, h_out, phi_out};
    for (const void* q : ptrs)
        if (!aligned16(q)) return fail(M3_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
    const int64_t units = dims->batch * dims->nheads, N = dims->dstate, P = dims->headdim;
    const SegSrc src{seg->h, units * N * P, N * P, seg->phi, units * (N / 2), N / 2,
                     seg->lam_sum, units, 1};
    cudaError_t e = launch_state_combine(units, static_cast<int>(N), static_cast<int>(P), nseg, src,
                                         h_out, phi_out, nullptr, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "state combine launch");
    return M3_OK;
}

m3_status m3_decode_step_proj(const m3_dims* dims, const m3_inputs* in, const m3_proj* proj,
                              const m3_state* state_in, const m3_state* state_out, void* o,
                              void* stream) {
    if (!proj) return fail(M3_ERR_INVALID_ARG, "proj is NULL");
    return decode_impl(dims, in, proj, state_in, state_out, o, stream);
}

m3_status m3_scan_check(void* workspace) {
    if (!workspace) return fail(M3_ERR_INVALID_ARG, "workspace is NULL");
    int32_t w = 0;
    cudaError_t e = cudaMemcpy(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "status read");
    if (w == 0) return M3_OK;
    // Re-arm the workspace: zero the whole header so the next call starts clean.
    e = cudaMemset(workspace, 0, kWsHeader);
    if (e != cudaSuccess) return cuda_fail(e, "status reset");
    return fail(M3_ERR_TIMEOUT, "a bounded wait between CTAs gave up (code %d)", w);
}

const char* m3_status_str(m3_status s) {
    switch (s) {
        case M3_OK: return "ok";
        case M3_ERR_INVALID_ARG: return "invalid argument";
        case M3_ERR_UNSUPPORTED: return "unsupported shape";
        case M3_ERR_CUDA: return "CUDA error";
        case M3_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

const char* m3_last_error(void) { return g_err; }

}  // extern "C"

extern "C" {

// The backward's workspace: the status header, the sequential form's intermediate buffers,
// then (where the chunked tensor-core form runs) its chunk states.
static size_t bwd_simt_bytes(const m3_dims* dims) {
    return sizeof(float) * scan_bwd_workspace_floats(dims->batch, dims->seqlen, dims->nheads,
                                                     dims->dstate, dims->rank);
}
static bool bwd_uses_tc(const m3_dims* dims, const m3::ScanParams& p) {
    return !(dims->flags & M3_BWD_FP32) && bwd_tc_supported(p, dims->in_dtype == M3_BF16);
}

size_t m3_scan_bwd_workspace_bytes(const m3_dims* dims) {
    if (check_dims(dims, false) != M3_OK) return 0;
    m3_inputs none{};
    const ScanParams p = make_params(dims, &none, nullptr, nullptr, nullptr);
    size_t n = kWsHeader + (bwd_simt_bytes(dims) + 255) / 256 * 256;
    if (bwd_uses_tc(dims, p)) n += bwd_tc_workspace_bytes(p);
    return n;
}

m3_status m3_scan_bwd(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                      const void* dy, const m3_state_grad* dfinal, const m3_grads* grads,
                      const m3_state_grad* dinit, void* workspace, size_t ws_bytes,
                      void* stream) {
    g_err[0] = 0;
    m3_status st = check_dims(dims, false);
    if (st != M3_OK) return st;
    const bool any = dims->batch * dims->seqlen * dims->nheads > 0;
    if ((st = check_inputs(in, any)) != M3_OK) return st;
    if ((st = check_state(init, "initial")) != M3_OK) return st;
    if (!grads) return fail(M3_ERR_INVALID_ARG, "grads is NULL");
    if (any) {
        const void* req[] = {dy, grads->dx, grads->dB, grads->dC, grads->dtheta,
                             grads->ddt, grads->dA, grads->dlam};
        const char* names[] = {"dy", "dx", "dB", "dC", "dtheta", "ddt", "dA", "dlam"};
        for (int i = 0; i < 8; ++i) {
            if (!req[i]) return fail(M3_ERR_INVALID_ARG, "%s is NULL", names[i]);
            if (!aligned16(req[i]))
                return fail(M3_ERR_INVALID_ARG, "%s is not 16-byte aligned", names[i]);
        }
    }
    const void* opt[] = {grads->dB_bias, grads->dC_bias, grads->ddt_bias,
                         dfinal ? dfinal->h : nullptr, dfinal ? dfinal->phi : nullptr,
                         dfinal ? dfinal->prev_B : nullptr, dfinal ? dfinal->prev_x : nullptr,
                         dinit ? dinit->h : nullptr, dinit ? dinit->phi : nullptr,
                         dinit ? dinit->prev_B : nullptr, dinit ? dinit->prev_x : nullptr};
    for (const void* q : opt)
        if (q && !aligned16(q))
            return fail(M3_ERR_INVALID_ARG, "gradient pointers must be 16-byte aligned");
    const size_t smem = scan_bwd_smem_bytes(dims->dstate, dims->headdim, dims->rank);
    if (smem > 227 * 1024)
        return fail(M3_ERR_UNSUPPORTED, "backward needs %zu bytes of shared memory", smem);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t H = dims->nheads, R = dims->rank, N = dims->dstate, P = dims->headdim;
    const int64_t units = dims->batch * H;
    if (!any) {
        // no token: the biases get nothing and the initial state's gradient is the final one's
        cudaError_t e = cudaSuccess;
        if (grads->dB_bias) e = cudaMemsetAsync(grads->dB_bias, 0, H * R * N * 4, s);
        if (e == cudaSuccess && grads->dC_bias) e = cudaMemsetAsync(grads->dC_bias, 0, H * R * N * 4, s);
        if (e == cudaSuccess && grads->ddt_bias) e = cudaMemsetAsync(grads->ddt_bias, 0, H * 4, s);
        float* dst[4] = {dinit ? dinit->h : nullptr, dinit ? dinit->phi : nullptr,
                         dinit ? dinit->prev_B : nullptr, dinit ? dinit->prev_x : nullptr};
        const float* src[4] = {dfinal ? dfinal->h : nullptr, dfinal ? dfinal->phi : nullptr,
                               dfinal ? dfinal->prev_B : nullptr, dfinal ? dfinal->prev_x : nullptr};
        const size_t bytes[4] = {static_cast<size_t>(units * N * P * 4),
                                 static_cast<size_t>(units * (N / 2) * 4),
                                 static_cast<size_t>(units * R * N * 4),
                                 static_cast<size_t>(units * R * P * 4)};
        for (int i = 0; i < 4 && e == cudaSuccess; ++i) {
            if (!dst[i] || bytes[i] == 0) continue;
            e = src[i] ? cudaMemcpyAsync(dst[i], src[i], bytes[i], cudaMemcpyDeviceToDevice, s)
                       : cudaMemsetAsync(dst[i], 0, bytes[i], s);
        }
        return e == cudaSuccess ? M3_OK : cuda_fail(e, "empty-sequence gradient copy");
    }
    const size_t need = m3_scan_bwd_workspace_bytes(dims);
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || ws_bytes < need)
        return fail(M3_ERR_INVALID_ARG, "workspace: NULL, misaligned or below %zu bytes", need);
    ScanParams p = make_params(dims, in, init, nullptr, nullptr);
    BwdGrads g{};
    g.dy = dy;
    if (dfinal) { g.dh1 = dfinal->h; g.dphi1 = dfinal->phi; g.dprevB1 = dfinal->prev_B; g.dprevx1 = dfinal->prev_x; }
    g.dx = grads->dx; g.dB = grads->dB; g.dC = grads->dC; g.dtheta = grads->dtheta;
    g.ddt = grads->ddt; g.dA = grads->dA; g.dlam = grads->dlam;
    g.dBbias = grads->dB_bias; g.dCbias = grads->dC_bias; g.ddtbias = grads->ddt_bias;
    if (dinit) { g.dh0 = dinit->h; g.dphi0 = dinit->phi; g.dprevB0 = dinit->prev_B; g.dprevx0 = dinit->prev_x; }
    char* ws = static_cast<char*>(workspace);
    int32_t* status = reinterpret_cast<int32_t*>(ws);
    void* tc_ws = bwd_uses_tc(dims, p) ? ws + kWsHeader + (bwd_simt_bytes(dims) + 255) / 256 * 256
                                       : nullptr;
    p.status = status;
    cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (e == cudaSuccess)
        e = launch_scan_bwd(p, g, dims->in_dtype == M3_BF16,
                            reinterpret_cast<float*>(ws + kWsHeader), tc_ws, status, s);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    return M3_OK;
}

}  // extern "C"
