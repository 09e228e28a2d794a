// fa_lib.cu -- the library is built as one translation unit so that every
// kernel shares the device error word without relocatable device code.
#include "fa_api.cu"
#include "prefill_sm100.cu"
#include "decode_tc_sm100.cu"
#include "decode_sm100.cu"
#include "decode_noalloc.cu"
#include "bwd_sm100.cu"
#include "fp8_prep.cu"
