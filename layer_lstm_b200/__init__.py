"""B200-native multi-layer / bidirectional LSTM forward and BPTT.

The compute path is the C-ABI library ``liblstm_b200.so`` (declared in
``include/lstm.h``); ``layer_lstm_b200.binding`` marshals arguments to it.
Importing this package does not load the library; ``binding.load()`` does.
"""
__all__ = ["binding", "workloads"]
