// gq_psgd.h -- internal interface of the PowerSGD low-rank kernels (gq_psgd.cu)
// used by the host side of the C ABI.
#ifndef GQ_PSGD_H
#define GQ_PSGD_H

#include "gq_internal.h"

namespace gq {

// PowerSGD low-rank step: the matrices of one launch (at most kPsgdGroup), each
// n x m row-major, stored back to back per worker.
constexpr int kPsgdGroup = 64;
struct PsgdArgs {
    const float* g;   // [W][total] gradients (project)
    float* m;         // [W][total] state: M_prev (or E) in, M out (project); M (back)
    const float* p;   // [ptotal] P_hat: previous (project), current (back, reconstruct)
    const float* q;   // [qtotal] Q: warm start (project), mean (reconstruct)
    float* pw;        // [W][ptotal] P_w (project)
    float* psum;      // [ptotal] summed P, orthonormalized in place (orth)
    float* qpart;     // [chunks][W][qtotal] row-chunk partials (back)
    float* qw;        // [W][qtotal] Q_w (back reduce)
    float* out;       // [total] Ghat (reconstruct)
    long long total, ptotal, qtotal;  // elements per worker: sum n m, sum n r, sum m r
    int W;
    int rank;
    int have_prev;
    int chunk_rows;  // rows per back-projection chunk
    int count;       // matrices in this launch
    int rows[kPsgdGroup], cols[kPsgdGroup];
    long long goff[kPsgdGroup], poff[kPsgdGroup], qoff[kPsgdGroup];
    long long tile0[kPsgdGroup + 1];  // first work tile of each matrix; tile0[count] = total
};

cudaError_t launch_psgd_project(const PsgdArgs& a, bool vec, int sms, cudaStream_t st);
cudaError_t launch_psgd_orth(const PsgdArgs& a, cudaStream_t st);
size_t psgd_back_smem(int rank, int chunk_rows, bool vec);
cudaError_t launch_psgd_back(const PsgdArgs& a, bool vec, int sms, cudaStream_t st);
cudaError_t launch_psgd_back_reduce(const PsgdArgs& a, int sms, cudaStream_t st);
cudaError_t launch_psgd_mean(const float* qsum, float* q, long long len, int W, int sms,
                             cudaStream_t st);
cudaError_t launch_psgd_reconstruct(const PsgdArgs& a, bool vec, int sms, cudaStream_t st);
// Every m a multiple of 4; tiles of (matrix, 1024 columns, 128 rows).
cudaError_t launch_psgd_reconstruct_cols(const PsgdArgs& a, int sms, cudaStream_t st);

}  // namespace gq

#endif  // GQ_PSGD_H
