// kvq_srft_d96.cu -- the SRFT codec kernels at D = 96 (see kvq_srft.cuh).
#define KVQ_SRFT_D 96
#include "kvq_srft.cuh"
