// Single translation unit of libinstagen.so (the kernels share one device
// error word, so they are compiled together without relocatable device code).
#include "permute.cu"
#include "kmeans.cu"
#include "select.cu"
#include "pqvote.cu"
#include "attention.cu"
#include "api.cu"
#include "cluster_static.cu"
