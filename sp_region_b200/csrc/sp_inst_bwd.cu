// Instantiations of the fast backward kernel k_bwd_tma for one (I/O dtype,
// norm) pair, chosen at compile time: SP_T_BF16 (0: fp32, 1: bf16) and SP_LN
// (0: RMSNorm, 1: LayerNorm).  The build compiles this file once per pair, in
// parallel, and links the four objects into the library.
#include "sp_bwd.cuh"
#include "sp_plans.h"

#if !defined(SP_T_BF16) || !defined(SP_LN)
#error "compile with -DSP_T_BF16=0|1 -DSP_LN=0|1"
#endif

#define SP_CAT2(a, b) a##b
#define SP_CAT(a, b) SP_CAT2(a, b)
#if SP_T_BF16
#define SP_TAG_T bf16
#else
#define SP_TAG_T f32
#endif
#if SP_LN
#define SP_TAG SP_CAT(SP_TAG_T, _ln)
#else
#define SP_TAG SP_CAT(SP_TAG_T, _rms)
#endif

namespace spk {
namespace {

using T = typename std::conditional<SP_T_BF16, __nv_bfloat16, float>::type;
constexpr bool LN = SP_LN != 0;

#define SP_BWD_CASE(ID)                                                                 \
    case ID:                                                                            \
        return (const void*)k_bwd_tma<T, kBwdPlans[ID].V, kBwdPlans[ID].G,              \
                                      kBwdPlans[ID].maxT, LN, kBwdPlans[ID].acc, EXACT>;

template <bool EXACT>
const void* bwd_kernel(int id)
{
    static_assert(kNumBwdPlans == 24, "one case per backward plan");
    switch (id) {
        SP_BWD_CASE(0) SP_BWD_CASE(1) SP_BWD_CASE(2) SP_BWD_CASE(3) SP_BWD_CASE(4)
        SP_BWD_CASE(5) SP_BWD_CASE(6) SP_BWD_CASE(7) SP_BWD_CASE(8) SP_BWD_CASE(9)
        SP_BWD_CASE(10) SP_BWD_CASE(11) SP_BWD_CASE(12) SP_BWD_CASE(13) SP_BWD_CASE(14)
        SP_BWD_CASE(15) SP_BWD_CASE(16) SP_BWD_CASE(17) SP_BWD_CASE(18) SP_BWD_CASE(19)
        SP_BWD_CASE(20) SP_BWD_CASE(21) SP_BWD_CASE(22) SP_BWD_CASE(23)
    }
    return nullptr;
}

}  // namespace

const void* SP_CAT(bwd_kernel_, SP_TAG)(int id, bool exact)
{
    return exact ? bwd_kernel<true>(id) : bwd_kernel<false>(id);
}

SPK_ERROR_WORD_ACCESSOR(SP_CAT(error_word_bwd_, SP_TAG))

}  // namespace spk
