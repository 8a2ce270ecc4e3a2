// fa_lib.cu - single translation unit of libfa_b200.so.  The kernels share one
// device error word, so the library is compiled as one unit instead of with
// relocatable device code.
#include "fa_api.cu"
#include "fa_fwd.cu"
#include "fa_bwd.cu"
#include "fa_decode.cu"
#include "fa_decode_static.cu"
#include "fa_selftest.cu"
