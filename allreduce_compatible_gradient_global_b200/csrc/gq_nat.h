// gq_nat.h -- launch arguments of the natural-compression kernels (gq_nat.cu).
#ifndef GQ_NAT_H
#define GQ_NAT_H

#include "gq_internal.h"

namespace gq {

constexpr unsigned kFlagNonfiniteNat = 8u;  // natural compression met inf / NaN
constexpr uint32_t kNatTag = 0x4E410000u;   // Philox key word 1 is seed_hi ^ kNatTag

struct NatArgs {
    const float* x;                 // quantize: [W][n] input
    unsigned short* codes;          // quantize: [W][n] codes
    const unsigned short* ccodes;   // decode: [W][n] codes
    float* out;                     // decode: [n] sum over workers
    long long n;                    // coordinates per worker
    int W;
    unsigned int worker0;           // Philox worker index of row 0
    unsigned int step;
    const unsigned int* step_dev;   // non-null: the step is read here, not from `step`
    RoundKeys rk;
    WsHeader* hdr;
};

cudaError_t launch_nat_quantize(const NatArgs& a, bool vec, int sms, cudaStream_t st);
cudaError_t launch_nat_decode_sum(const NatArgs& a, bool vec, int sms, cudaStream_t st);

}  // namespace gq

#endif  // GQ_NAT_H
