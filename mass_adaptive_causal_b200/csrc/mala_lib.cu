// mala_lib.cu -- the whole CUDA library as one translation unit, so that the
// device status word (common.cuh) exists once per GPU and every kernel can
// set it without relocatable device code.
#include "api.cuh"
