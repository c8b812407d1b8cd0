// kvq_srft_d64.cu -- the SRFT codec kernels at D = 64 (see kvq_srft.cuh).
#define KVQ_SRFT_D 64
#include "kvq_srft.cuh"
