// producer.cuh -- arguments and host entry points of the write-term producer (producer.cu).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace prism {

// One call: B x H sequences of T tokens, width d (64 or 128), L ranks.  Layouts as in prism.h:
// x, v [B,T,H,d] bf16; conv [H,4,d] fp32; Wk, Wp [H,L,d,d] bf16 (row = output index);
// beta [B,T,H,L] fp32; u, w [B,T,H,L,d] bf16.
struct ProducerArgs {
    int B, H, T, d, L;
    const void *x, *v;
    const float *conv;
    const void *Wk, *Wp;
    const float *beta;
    void *u, *w;
    int stall;  // the give-up test: no weight load is issued, every wait runs out after a short limit
};

cudaError_t launch_write_producer(const ProducerArgs &a, cudaStream_t s);
cudaError_t producer_status(uint32_t *out);  // read and clear the producer's status word

}  // namespace prism
