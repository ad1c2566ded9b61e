// Plan tables of the fast streaming kernels, shared by the host planner
// (sp_region.cu) and the translation units that instantiate the kernels
// (sp_inst_fwd.cu, sp_inst_bwd.cu), plus the accessors those units export.
#pragma once

namespace spk {

// ---------------------------------------------------------------------------
// Fast-kernel plans: V vectors of 8 features per consumer thread, G consumer
// groups (each takes every G-th row of the CTA), at most maxT threads (which
// sets the register budget), and for the backward the parameter-gradient
// partials in registers or shared memory.  A group needs
// C = 32 * ceil(ceil(hv / V) / 32) threads; a launch has G*C + 32.
// ---------------------------------------------------------------------------
struct Plan {
    int V, G, maxT;
    int acc;   // backward parameter-gradient partials: 0 registers, 1 shared, 2 tensor memory
    int CS;   // CTAs per token row (a thread-block cluster when 2)
};

constexpr Plan kFwdPlans[] = {
    {1, 1, 1024, 0, 1},   // 0
    {1, 2, 800, 0, 1},    // 1
    {1, 4, 1024, 0, 1},   // 2
    {2, 1, 544, 0, 1},    // 3
    {2, 2, 800, 0, 1},    // 4
    {3, 1, 544, 0, 1},    // 5
    {3, 2, 800, 0, 1},    // 6
    {4, 1, 544, 0, 1},    // 7
    {4, 2, 800, 0, 1},    // 8
    {2, 3, 800, 0, 1},    // 9
    {4, 4, 544, 0, 1},    // 10
    {4, 6, 800, 0, 1},    // 11
    {3, 3, 800, 0, 1},    // 12
    {4, 4, 800, 0, 1},    // 13
    {1, 2, 800, 0, 2},    // 14
    {2, 2, 800, 0, 2},    // 15
    {2, 1, 544, 0, 2},    // 16
    {1, 1, 1024, 0, 2},   // 17
    {4, 1, 544, 0, 2},    // 18
};
constexpr Plan kBwdPlans[] = {
    {1, 1, 1024, 0, 1},   // 0
    {1, 1, 800, 0, 1},    // 1
    {1, 2, 800, 0, 1},    // 2
    {2, 1, 544, 1, 1},     // 3
    {2, 1, 800, 0, 1},    // 4
    {3, 1, 544, 1, 1},     // 5
    {4, 1, 544, 1, 1},     // 6
    {2, 1, 544, 0, 1},    // 7
    {2, 2, 800, 1, 1},     // 8
    {3, 2, 800, 1, 1},     // 9
    {4, 2, 800, 1, 1},     // 10
    {2, 3, 800, 1, 1},     // 11
    {4, 4, 544, 1, 1},     // 12
    {3, 3, 800, 1, 1},     // 13
    {4, 4, 800, 1, 1},     // 14
    {2, 2, 800, 2, 1},        // 15
    {3, 2, 800, 2, 1},        // 16
    {3, 1, 544, 2, 1},        // 17
    {2, 1, 800, 2, 1},        // 18
    {4, 4, 544, 2, 1},        // 19
    {2, 3, 800, 2, 1},        // 20
    {4, 1, 544, 2, 1},        // 21
    {2, 1, 544, 2, 1},        // 22
    {4, 2, 544, 2, 1},        // 23
};
constexpr int kNumFwdPlans = sizeof(kFwdPlans) / sizeof(kFwdPlans[0]);
constexpr int kNumBwdPlans = sizeof(kBwdPlans) / sizeof(kBwdPlans[0]);

// Kernel of fast-kernel plan `id` (forward or backward table), for the I/O
// dtype and norm of the unit that defines it; exact: the threads' vectors
// tile the row exactly.  One accessor per (dtype, norm) unit.
const void* fwd_kernel_bf16_ln(int id, bool exact);
const void* fwd_kernel_bf16_rms(int id, bool exact);
const void* fwd_kernel_f32_ln(int id, bool exact);
const void* fwd_kernel_f32_rms(int id, bool exact);
const void* bwd_kernel_bf16_ln(int id, bool exact);
const void* bwd_kernel_bf16_rms(int id, bool exact);
const void* bwd_kernel_f32_ln(int id, bool exact);
const void* bwd_kernel_f32_rms(int id, bool exact);

// Every translation unit with kernels has its own device error word; these
// read (and optionally clear) the word of one unit.  0 on success.
int error_word_host(unsigned* v, int clear);
int error_word_gemm(unsigned* v, int clear);
int error_word_fwd_bf16_ln(unsigned* v, int clear);
int error_word_fwd_bf16_rms(unsigned* v, int clear);
int error_word_fwd_f32_ln(unsigned* v, int clear);
int error_word_fwd_f32_rms(unsigned* v, int clear);
int error_word_bwd_bf16_ln(unsigned* v, int clear);
int error_word_bwd_bf16_rms(unsigned* v, int clear);
int error_word_bwd_f32_ln(unsigned* v, int clear);
int error_word_bwd_f32_rms(unsigned* v, int clear);

}  // namespace spk
