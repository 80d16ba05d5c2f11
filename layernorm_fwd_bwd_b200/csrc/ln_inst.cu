// ln_inst.cu -- one instantiation unit of the dispatch templates
// (ln_dispatch.cuh).  The build compiles this file once per combination of
//   LN_INST_DIR   0 forward, 1 backward
//   LN_INST_T     0 fp32, 1 bf16, 2 fp16
//   LN_INST_MODE  the variant (forward: lnk::kFwdResidual; backward: any
//                 combination of lnk::kBwdAccumulate and lnk::kBwdRecompute)
// into its own object, so the kernels of the combinations compile in
// parallel; ln_api.cu calls the instantiations.
#include "ln_dispatch.cuh"

#if !defined(LN_INST_DIR) || !defined(LN_INST_T) || !defined(LN_INST_MODE)
#error "compile with -DLN_INST_DIR=.. -DLN_INST_T=.. -DLN_INST_MODE=.."
#endif

#if LN_INST_T == 0
#define LN_INST_TYPE float
#elif LN_INST_T == 1
#define LN_INST_TYPE lnk::bf16
#elif LN_INST_T == 2
#define LN_INST_TYPE lnk::f16
#else
#error "LN_INST_T: 0 (fp32), 1 (bf16) or 2 (fp16)"
#endif

#if LN_INST_DIR == 0
template int lnh::fwd_dispatch<LN_INST_TYPE, LN_INST_MODE>(const lnh::FwdArgs &);
#else
template int lnh::bwd_dispatch<LN_INST_TYPE, LN_INST_MODE>(const lnh::BwdArgs &);
#endif
