// sa_status_codes.h - numeric status codes shared by host and device code.
// They equal the sa_status values of include/sparse_attn.h.
#pragma once

#define SA_STATUS_OK 0
#define SA_STATUS_INVALID_ARG 1
#define SA_STATUS_UNSUPPORTED 2
#define SA_STATUS_CUDA 3
#define SA_STATUS_TIMEOUT 4
#define SA_STATUS_DEVICE_ASSERT 5
