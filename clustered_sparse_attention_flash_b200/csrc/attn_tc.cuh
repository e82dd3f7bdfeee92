// Tensor-core (tcgen05 / TMEM) hybrid attention for bf16; see attn_tc.cu.
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace svg {
constexpr int kMaxCkBits = 4096;
bool attn_tc_supported(int d, int Ck);
// The next attention launch on this host thread records `begin` and `end`
// around the attention kernel alone; attn_tc_kernel_was_timed() reports
// whether a launch used them since.
void attn_tc_time_next_kernel(cudaEvent_t begin, cudaEvent_t end);
bool attn_tc_kernel_was_timed();
size_t attn_tc_ws_bytes(int H, int Nq, int Nk, int d, int Cq, int Ck);
cudaError_t attn_tc_run(const void* Qp, const void* Kp, const void* Vp, const int32_t* q_off,
                        const int32_t* k_off, const int32_t* perm_q, const float* Kbar,
                        const float* Vbar, const int32_t* sel, const int32_t* n_sel, int H, int Nq,
                        int Nk, int d, int Cq, int Ck, float scale, void* O, void* ws,
                        cudaStream_t st);
}  // namespace svg
