// Internal declarations shared by the host entry points and the kernel files.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include <utility>

#include "../../include/m3.h"

namespace m3 {

// Everything a scan or decode launch needs, already validated by the host entry point.
struct ScanParams {
    int64_t b, L, H, G, P, N, R, Q;
    int32_t bc_norm;
    float eps;
    const void* x;
    const void* B;
    const void* C;
    const void* theta;
    const float* dt;
    const float* A;
    const float* lam;
    const float* Bbias;  // may be null
    const float* Cbias;  // may be null
    const float* dt_bias;  // [H], may be null; read only with M3_DT_SOFTPLUS
    uint32_t flags;        // M3_DT_SOFTPLUS | M3_LAM_SIGMOID
    // decode with the MIMO projections (m3_decode_step_proj): x' and z' [b,H,P], the per-head
    // weights [H,R,P]; y then receives O' [b,H,P]
    int32_t proj;
    const void* xprj;
    const void* zprj;
    const float* WX;
    const float* WZ;
    const float* WO;
    // initial state; all null = zero state
    const float* h0;
    const float* phi0;
    const void* prevB0;
    const void* prevx0;
    // final state; all null = not written
    float* h1;
    float* phi1;
    void* prevB1;
    void* prevx1;
    void* y;
    int32_t* status;  // device status word (workspace), may be null for decode
    // Test hook of the tensor-core scans: > 0 makes CTA 0 skip the theta load of that chunk,
    // so that its bounded wait runs out and the timeout path (status word, drain, TMEM
    // release) is exercised. Set only from the M3_TEST_SKIP_THETA_LOAD environment variable.
    int32_t test_skip_theta;
    void* ws;         // workspace base
    size_t ws_bytes;
};

// Launchers. Each returns cudaSuccess or the launch error; none synchronises.
cudaError_t launch_decode(const ScanParams& p, bool bf16, cudaStream_t s);
// Shared-memory bytes the SIMT scan needs for these dims (0 = cannot run).
size_t simt_scan_smem_bytes(const ScanParams& p);
cudaError_t launch_scan_simt(const ScanParams& p, bool bf16, cudaStream_t s);
// Warp-specialised tensor-core scan (bf16, N = 128, P = 64, chunk * R = 128, R <= 4): one
// CTA per (batch, head) unit and SM; its workspace body holds the fp32 RMS scales.
bool pipe_scan_supported(const ScanParams& p, bool bf16);
size_t pipe_scan_workspace_bytes(const ScanParams& p);
cudaError_t launch_scan_pipe(const ScanParams& p, void* ws_body, size_t body_bytes, cudaStream_t s);
// Tensor-core scan (bf16, N = 128, P = 64, chunk * R = 64).
bool tc_scan_supported(const ScanParams& p, bool bf16);
// Workspace bytes the tensor-core scan needs beyond the status header: with the end states of
// the sequence-parallel form's segments (preferred), or without them (minimum: one segment).
size_t tc_scan_workspace_bytes(const ScanParams& p);
size_t tc_scan_workspace_min_bytes(const ScanParams& p);
// ws_body: the workspace after the status header, body_bytes long (at least the minimum); the
// scan uses as many segments as the preferred plan has and body_bytes holds.
cudaError_t launch_scan_tc(const ScanParams& p, void* ws_body, size_t body_bytes, cudaStream_t s);
// The state-only pass over the whole sequence of every unit (m3_scan_state): the end state h,
// the angle and the summed log-decay go to out_h [units][N][P], out_phi [units][N/2],
// out_lam [units].
cudaError_t launch_scan_state_tc(const ScanParams& p, void* ws_body, size_t body_bytes,
                                 float* out_h, float* out_phi, float* out_lam, cudaStream_t s);
// Where the segment states for a combine live: element strides between segments and units.
struct SegSrc {
    const float* h;
    int64_t h_seg, h_unit;
    const float* phi;
    int64_t phi_seg, phi_unit;
    const float* lam;
    int64_t lam_seg, lam_unit;
};
// nseg segment states -> the state after the last of them (h_out [units][N][P], phi_out
// [units][N/2]) and, if lam_out is set, their summed log-decay [units].
cudaError_t launch_state_combine(int64_t units, int N, int P, int nseg, const SegSrc& src,
                                 float* h_out, float* phi_out, float* lam_out, cudaStream_t s);
// The smallest workspace m3_scan_fwd's work runs in (one segment per sequence), and the scan
// entry point with that lower bound instead of m3_scan_workspace_bytes (for the fixed scratch
// of m3_scan_fwd_noalloc).
size_t scan_workspace_min_bytes(const m3_dims* dims);
m3_status scan_fwd_with(const m3_dims* dims, const m3_inputs* in, const m3_state* init,
                        const m3_state* final_state, void* y, void* workspace, size_t ws_bytes,
                        size_t need, void* stream);
// Records msg as this thread's m3_last_error() text and returns s.
m3_status set_error(m3_status s, const char* msg);
// The per-token RMS scales of B and C for the tensor-core scans: out[((b * G + g) * Lpad + l)
// * R + r] = (1 / rms(B row), 1 / rms(C row)), Lpad = L rounded up to whole chunks of Q tokens.
// The kernel lets a scan launched with launch_after_rms start before it finishes.
cudaError_t launch_rms_scales(const ScanParams& p, int64_t Q, float2* out, cudaStream_t s);
// Launches kernel<<<grid, block, smem, s>>>(args...) so that it may start while the kernel
// before it in the stream (the RMS scales) finishes; the kernel must call grid_dep_wait()
// before it reads that kernel's output.
template <typename... KArgs, typename... Args>
cudaError_t launch_after_rms(void (*kernel)(KArgs...), unsigned grid, unsigned block,
                             size_t smem, cudaStream_t s, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}
// SM count of the calling thread's current device, looked up once per device (148, the
// B200's count, when no device answers). Safe to call from several host threads.
int device_sm_count();
// Persistent decode with bulk asynchronous copies (bf16, N * P <= 8192).
bool decode_bulk_supported(const ScanParams& p, bool bf16);
size_t decode_bulk_smem_bytes(const ScanParams& p);
cudaError_t launch_decode_bulk(const ScanParams& p, cudaStream_t s);
// Decode with the rank-2R update and the readout on the tensor cores (bf16, N = 128, P = 64).
bool decode_tc_supported(const ScanParams& p, bool bf16);
cudaError_t launch_decode_tc(const ScanParams& p, cudaStream_t s);
// Size of the decode kernel's dynamic shared memory for these dims.
size_t decode_smem_bytes(const ScanParams& p);

// Backward pass of the scan (m3_scan_bwd): the output and final-state gradients in, the input
// and initial-state gradients out (all fp32; the nullable ones as in m3.h).
struct BwdGrads {
    const void* dy;
    const float* dh1;
    const float* dphi1;
    const float* dprevB1;
    const float* dprevx1;
    float* dx;
    float* dB;
    float* dC;
    float* dtheta;
    float* ddt;
    float* dA;
    float* dlam;
    float* dBbias;
    float* dCbias;
    float* ddtbias;
    float* dh0;
    float* dphi0;
    float* dprevB0;
    float* dprevx0;
};
// Tokens per staged chunk of the backward sweeps, their workspace (floats) and shared memory.
int bwd_chunk_tokens(int64_t R);
size_t scan_bwd_workspace_floats(int64_t b, int64_t L, int64_t H, int64_t N, int64_t R);
size_t scan_bwd_smem_bytes(int64_t N, int64_t P, int64_t R);
// f: the forward's inputs and initial state (validated); ws: scan_bwd_workspace_floats floats,
// 256-byte aligned. L >= 1 and b >= 1. tc_ws: bwd_tc_workspace_bytes more (256-byte aligned)
// when bwd_tc_supported, which then runs the chunked tensor-core backward; status: the
// device status word the tensor-core kernels set when a bounded wait gives up.
cudaError_t launch_scan_bwd(const ScanParams& f, const BwdGrads& g, bool bf16, float* ws,
                            void* tc_ws, int32_t* status, cudaStream_t s);

// Chunked backward on the tensor cores (bf16, R = 1, N = 128, P = 64, H % 4 == 0, without
// M3_BWD_FP32): the forward state pass, then one CTA per unit over its chunks in reverse.
bool bwd_tc_supported(const ScanParams& p, bool bf16);
size_t bwd_tc_workspace_bytes(const ScanParams& p);
// Where the chunked backward writes: the sequential backward's intermediate buffers (wdB,
// wdC [b,L,H,R,N], here as bf16; wsc [units][L][4], wprev [units][R][N], wF [units]) and the
// gradients it produces itself.
struct BwdTcOut {
    const void* dy;
    const float* dh1;
    const float* dphi1;
    const float* dprevx1;
    float* dx;
    float* dtheta;
    void* wdB;
    void* wdC;
    float* wsc;
    float* wprev;
    float* wF;
    float* dh0;
    float* dphi0;
    float* dprevx0;
    float* dBbias;
    float* dCbias;
    int32_t* status;
};
cudaError_t launch_bwd_tc(const ScanParams& p, const BwdTcOut& o, void* ws, cudaStream_t s);
// The tensor-core scan's state-only pass over whole sequences, for the backward: per unit
// and chunk, e^{cum_0} H0' (bf16 in the swizzled [n][p] operand layout, 16384 bytes) into
// chunk_h and the angle before the chunk into chunk_phi [64]; the final state into hfin
// [units][N][P], phifin [units][N/2], lamfin [units]. rs: the RMS-scale buffer or null.
cudaError_t launch_bwd_states_tc(const ScanParams& p, float2* rs, uint8_t* chunk_h,
                                 float* chunk_phi, float* hfin, float* phifin, float* lamfin,
                                 cudaStream_t s);
// cuTensorMapEncodeTiled for a bf16 (else fp32) tensor, 128-byte swizzle (else none), unit
// element strides; map points at a CUtensorMap.
bool encode_tmap(void* map, bool bf16, int rank, const void* base, const uint64_t* dims,
                 const uint64_t* strides, const uint32_t* box, bool swizzle128);

}  // namespace m3
