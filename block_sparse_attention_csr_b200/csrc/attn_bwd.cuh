// Block-sparse backward of Radial Attention on sm_100a (see radial_lib.cu).
#pragma once
