#pragma once
#include "pba_device.cuh"
