// kvq_srft_d128.cu -- the SRFT codec kernels at D = 128 (see kvq_srft.cuh).
#define KVQ_SRFT_D 128
#include "kvq_srft.cuh"
