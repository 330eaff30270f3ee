// dart_backward.cuh -- argument blocks and launchers of the backward kernels
// (sma_bwd.cu, ssd_scan_bwd.cu), used by the C ABI in dart_abi.cu.
#pragma once

#include "dart_common.cuh"

namespace dart {

struct SmaBwdArgs {
    int B, L, H, P, N, S, G;
    const void* Q; const void* E; const void* Cm; const void* dH;
    float g; const float* dy;               // dy: [B,L,H,P] gradient of the layer output
    float* dQ; float* dE; float* dCm; float* ddH; float* dg;   // outputs (fp32); dCm [B,L,G,N]
    int* status;
    // workspace views (set by launch_sma_bwd)
    float* pbuf; float* dsbuf;              // softmax weights and score gradients: [B,H,L,C] on CUDA
                                            // cores, [B,H,C,L] on the tensor cores
    float* dCh;                             // [B,L,H,N] per-head dC
    float* gpart;                           // [B,H,tiles] per-tile dg
};

struct ScanBwdArgs {
    int B, L, H, P, N, S, G;
    const void* x; const float* dt; const float* A; const void* Bm; const void* Cm;
    const float* init;      // nullable [B,H,N,P] initial state of the forward
    const float* states;    // [B,H,C,N,P] boundary states written by the forward
    const float* dy;        // [B,L,H,P] gradient of y_ssd
    const float* ddH;       // nullable [B,H,C,N,P] gradient of the chunk memories
    const float* dC_add;    // nullable [B,L,G,N]: added to dC (e.g. the SMA backward's part; may be dC)
    float* dx; float* ddt; float* dA; float* dB; float* dC;   // outputs (fp32); dB, dC [B,L,G,N]
    float* dinit;           // nullable [B,H,N,P] output
    int* status;
    // workspace views (set by launch_ssd_scan_bwd)
    float* gin;             // [B,H,C,N,P] dS[c], then the adjoint entering chunk c from later chunks
    float* asum;            // [B,H,C] chunk decay sums
    float* rect;            // [B,H,C,S] the chunk-local decay-gradient term per token (CUDA cores);
                            // [6][B,H,C,S] the per-token scalars u, v, q1, colsum and the rowsum
                            // parts of row blocks 0 and 1 (tensor cores)
    float* c0;              // [B,H,C] sum(Gin o h_in) (tensor cores)
    float* dBh; float* dCh; // [B,L,H,N] per-head dB, dC
    float* dApart;          // [B,H,C]
};

size_t sma_bwd_workspace_bytes(int B, int L, int H, int N, int S);
// sma_bwd_tc.cu: the tensor-core SMA backward (bf16, N = 128, P = 64, S a multiple of 128)
bool sma_bwd_tc_applicable(int N, int P, int S, dart_dtype dt);
int sma_bwd_tc_tiles(int B, int L, int H, int S);
cudaError_t launch_sma_bwd_tc(const SmaBwdArgs& a, cudaStream_t st);
cudaError_t launch_sma_bwd(SmaBwdArgs a, void* workspace, dart_dtype dt, cudaStream_t st);
size_t scan_bwd_workspace_bytes(int B, int L, int H, int N, int P, int S);
bool scan_bwd_supported(int N, int P, int S);
cudaError_t launch_ssd_scan_bwd(ScanBwdArgs a, void* workspace, dart_dtype dt, cudaStream_t st);
// ssd_scan_bwd_tc.cu: the intra-chunk products of the scan backward on the tensor cores
bool scan_bwd_tc_applicable(int N, int P, int S, dart_dtype dt);
cudaError_t launch_scan_bwd_quad_tc(const ScanBwdArgs& a, cudaStream_t st);
cudaError_t launch_scan_bwd_dS_tc(const ScanBwdArgs& a, cudaStream_t st);

}  // namespace dart
