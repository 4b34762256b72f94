// library.cu -- single translation unit for libgemma_attn.so, so that the device
// status word and every kernel live in one module without relocatable device code.
#include "api.cu"
#include "rope.cu"
#include "prefill.cu"
#include "decode.cu"
#include "decode_umma.cu"
#include "decode_noalloc.cu"
#include "append.cu"
#include "selftest.cu"
