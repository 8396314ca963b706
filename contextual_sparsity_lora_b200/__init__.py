"""B200-native (sm_100a) SparseLoRA hot path: a C-ABI CUDA library (libsparselora.so)
and its thin ctypes binding. Importing the package loads nothing; the binding
module loads the library on first use and raises if it is missing."""
